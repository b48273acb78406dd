"""Assemble test cases: joint-SVD factors, latent cache and current token.

Test infrastructure only.  Calls the seeded generators in ``synthetic`` for
random numbers and this package for every step of the method (joint SVD,
beta split, H2, latent, quantiser).  The arrays handed to the CUDA library
are the ones the oracle itself consumes: device-precision values are produced
here (float16 / bfloat16 rounding to nearest even, done with NumPy and plain
PyTorch CPU casts) and the oracle reads them back upcast to float64.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np
import torch

import synthetic
from oracle import qsvd_ref as ref
from oracle import quant_ref as qr


def to_device_dtype(a: np.ndarray, dtype: str) -> np.ndarray:
    """Round to the storage dtype; returns the raw array (float32, float16,
    or uint16 bit patterns for bfloat16)."""
    a32 = np.asarray(a, np.float64).astype(np.float32)
    if dtype == "f32":
        return a32
    if dtype == "f16":
        return a32.astype(np.float16)
    if dtype == "bf16":
        t = torch.from_numpy(np.ascontiguousarray(a32)).to(torch.bfloat16)
        return t.view(torch.int16).numpy().view(np.uint16)
    raise ValueError(dtype)


def from_device_dtype(a: np.ndarray, dtype: str) -> np.ndarray:
    """Values of a stored array as float64."""
    if dtype == "bf16":
        t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
        return t.to(torch.float64).numpy()
    return np.asarray(a).astype(np.float64)


def torch_dtype(dtype: str):
    return {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16,
            "i8": torch.int8, "i4": torch.uint8}[dtype]


def as_torch(a: np.ndarray, dtype: str) -> torch.Tensor:
    """Wrap a device-representation array as a CPU tensor of that dtype."""
    a = np.ascontiguousarray(a)
    if dtype == "bf16":
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
    return torch.from_numpy(a)


@dataclass
class Case:
    w: synthetic.Workload
    beta: float
    lengths: np.ndarray             # (B,) int32
    max_len: int
    # device representations
    wd_dev: np.ndarray              # E x r
    wuq_dev: np.ndarray             # r x E
    wuk_dev: np.ndarray
    wuv_dev: np.ndarray
    cache_dev: np.ndarray           # B x max_len x row (dtype-dependent)
    scales_dev: Optional[np.ndarray]  # B x max_len x r/group float16 (int caches)
    cnew: np.ndarray                # B x r float32 (current-token latent)
    # float64 values the oracle consumes
    wd: np.ndarray
    wuq: np.ndarray
    wuk: np.ndarray
    wuv: np.ndarray
    caches: List[np.ndarray] = field(default_factory=list)  # per b: len_b x r
    h2: Optional[np.ndarray] = None
    h2_q: Optional[np.ndarray] = None

    def reference(self) -> np.ndarray:
        """Oracle output (B x E) for this case, keys/values materialised."""
        rb = self.w.rope_base if self.w.rope else None
        return ref.decode_materialized(self.caches, self.lengths,
                                       self.cnew.astype(np.float64),
                                       self.wuq, self.wuk, self.wuv, self.w.H,
                                       rope_base=rb)


def compress(w: synthetic.Workload, r: Optional[int] = None,
             beta: Optional[float] = None, with_h2: bool = True):
    """Joint-SVD factors (float64) for a workload, optionally H2-rotated."""
    wq, wk, wv = synthetic.qkv_weights(w)
    u, s, vt = ref.joint_svd(wq, wk, wv)
    b = synthetic.beta(w) if beta is None else beta
    wd, wuq, wuk, wuv = ref.factors(u, s, vt, w.r if r is None else r, b)
    h2 = None
    if with_h2 and w.h2_n:
        h2 = ref.h2_matrix(w.h2_n, synthetic.small_orthogonal(w.h2_m))
        wd, wuq, wuk, wuv = ref.rotate_factors(wd, wuq, wuk, wuv, h2)
    return (wq, wk, wv), (u, s, vt), b, (wd, wuq, wuk, wuv), h2


def row_bytes(w: synthetic.Workload) -> int:
    return {"f32": 4 * w.r, "f16": 2 * w.r, "bf16": 2 * w.r, "i8": w.r,
            "i4": w.r // 2}[w.cache]


def build_case(w: synthetic.Workload, lengths: Optional[np.ndarray] = None,
               pad_rows: int = 20, pad_value: float = 3.0e4,
               factors_override=None) -> Case:
    """Full test case for workload ``w`` (sizes the oracle handles quickly).

    Rows of the cache at or past each sequence's length are filled with
    ``pad_value`` (a large finite number) so that a kernel that reads them
    into the softmax gives a visibly wrong answer."""
    if factors_override is None:
        _, _, b, (wd, wuq, wuk, wuv), h2 = compress(w)
    else:
        b, (wd, wuq, wuk, wuv), h2 = factors_override
    lens = synthetic.lengths(w) if lengths is None else np.asarray(lengths, np.int32)
    max_len = int(max(1, lens.max()) + pad_rows)
    wd_dev, wuq_dev, wuk_dev, wuv_dev = (to_device_dtype(m, w.weight)
                                         for m in (wd, wuq, wuk, wuv))
    wd_v, wuq_v, wuk_v, wuv_v = (from_device_dtype(m, w.weight)
                                 for m in (wd_dev, wuq_dev, wuk_dev, wuv_dev))
    B, r = w.B, w.r
    cnew = np.zeros((B, r), np.float32)
    caches = []
    is_int = w.cache in ("i4", "i8")
    if is_int:
        bits = 4 if w.cache == "i4" else 8
        codes_all = np.zeros((B, max_len, r), np.int8)
        scales = np.zeros((B, max_len, r // w.group), np.float16)
    else:
        pad = to_device_dtype(np.full((1,), pad_value), w.cache)[0]
        cache_dev = np.empty((B, max_len, r), dtype=to_device_dtype(np.zeros(1), w.cache).dtype)
        cache_dev[...] = pad
    for bi in range(B):
        n = int(lens[bi])
        x = synthetic.sequence_activations(w, bi, max(n, 1))
        c64 = ref.latent(x, wd_v)                  # n x r (float64)
        c32 = c64.astype(np.float32)
        cnew[bi] = c32[max(n, 1) - 1]
        if is_int:
            codes, sc, _ = qr.quantize(c32[:n], bits, w.group)
            codes_all[bi, :n] = codes
            scales[bi, :n] = sc
            # rows past the length: maximal codes with a large scale
            codes_all[bi, n:] = 5
            scales[bi, n:] = np.float16(1000.0)
            caches.append(qr.dequantize(codes, sc, w.group).astype(np.float64))
        else:
            dev = to_device_dtype(c64[:n], w.cache)
            cache_dev[bi, :n] = dev
            caches.append(from_device_dtype(dev, w.cache))
    if is_int:
        cache_dev = qr.pack_int4(codes_all) if w.cache == "i4" else codes_all
        scales_dev = scales
    else:
        scales_dev = None
    h2_q = synthetic.small_orthogonal(w.h2_m) if w.h2_n else None
    return Case(w=w, beta=b, lengths=lens, max_len=max_len, wd_dev=wd_dev,
                wuq_dev=wuq_dev, wuk_dev=wuk_dev, wuv_dev=wuv_dev,
                cache_dev=cache_dev, scales_dev=scales_dev, cnew=cnew,
                wd=wd_v, wuq=wuq_v, wuk=wuk_v, wuv=wuv_v, caches=caches,
                h2=h2, h2_q=h2_q)
