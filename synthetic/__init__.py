"""Seeded synthetic inputs for the joint-QKV latent decode path.

This module is the only code shared by the CPU oracle (``oracle/``) and the
CUDA library's tests and benchmark.  It draws random numbers with stated
distributions and shapes; it holds none of the method's arithmetic (no SVD,
no projection, no attention, no quantisation).

Workload shapes follow the five configurations this library is measured on:
a tiny case, LLaVA-v1.5-7B and 13B attention layers (E = 4096/5120 with
d_h = 128), and an int4/int8 latent cache.  The pages evaluate trained VLMs on
public benchmarks (ScienceQA, VizWiz, SEED-Bench, ...); none of that is here,
and these seeded inputs stand in for it.

Recipe (all generators are ``numpy.random.Generator(PCG64)`` seeded with
``[20251016 + 1000*cfg, stream]``, one independent stream per quantity):

* ``W_Q, W_K, W_V`` (E x E, fp32): ``U diag(sigma) V^T`` with Haar-random
  orthogonal ``U, V`` (QR of a Gaussian matrix, signs fixed by diag(R)) and a
  power-law spectrum ``sigma_i = kappa * i**-0.5`` (i = 1..E); ``kappa`` makes
  ``||W||_F^2 = E`` so query/key entries are O(1).
* ``X`` (tokens x E): i.i.d. N(0, 1); a seeded set of ``round(frac * E)``
  outlier channels (the same for every token) is multiplied by ``scale``.
* ``beta``: 0.5, or U(0.2, 0.8) for the 13B-shaped configuration.
* ragged lengths: integers uniform on an inclusive range.
* ``Q3``: the orthonormal 3x3 DCT-II matrix (deterministic), used as the small
  factor of the Kronecker rotation ``H_n (x) Q3``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Optional, Tuple

import numpy as np

BASE_SEED = 20251016

# one independent sub-stream per quantity
STREAM = {
    "wq": 1, "wk": 2, "wv": 3, "x": 4, "outliers": 5, "lengths": 6,
    "beta": 7, "xnew": 8, "direct_c": 9, "direct_w": 10, "direct_cnew": 11,
    "misc": 12,
}


@dataclass(frozen=True)
class Workload:
    """Shapes and dtypes of one configuration of the decode path."""
    name: str
    E: int
    H: int
    d_h: int
    r: int
    B: int
    L: int                         # tokens per sequence (max of the range if ragged)
    cache: str                     # "f32" | "f16" | "bf16" | "i8" | "i4"
    weight: str                    # "f32" | "f16" | "bf16"
    rope: bool
    beta: float = 0.5
    beta_range: Optional[Tuple[float, float]] = None
    outlier_frac: float = 0.01
    outlier_scale: float = 20.0
    group: int = 128
    h2_n: int = 0                  # Hadamard order of H2 = H_n (x) Q_m (0: no H2)
    h2_m: int = 0
    ragged: Optional[Tuple[int, int]] = None   # inclusive length range
    rope_base: float = 10000.0
    cfg_id: int = 0

    @property
    def seed(self) -> int:
        return BASE_SEED + 1000 * self.cfg_id


CONFIGS = {
    # tiny: one decode step, fp32 latent, absorbed mode
    0: Workload("tiny-fp32-absorbed", E=256, H=4, d_h=64, r=96, B=1, L=128,
                cache="f32", weight="f32", rope=False, outlier_frac=0.02,
                outlier_scale=20.0, cfg_id=0),
    # LLaVA-v1.5-7B attention layer, fp16 latent, absorbed query
    1: Workload("llava7b-fp16-absorbed", E=4096, H=32, d_h=128, r=1536, B=16,
                L=8192, cache="f16", weight="f16", rope=False, cfg_id=1),
    # same shapes, bf16 latent, RoPE on reconstructed keys
    2: Workload("llava7b-bf16-rope", E=4096, H=32, d_h=128, r=1536, B=16,
                L=8192, cache="bf16", weight="bf16", rope=True, cfg_id=2),
    # W8A4-style: int4 latent (groups of 128, fp16 scales), H2 = H_256 (x) Q3
    3: Workload("llava7b-int4-h2", E=4096, H=32, d_h=128, r=768, B=32,
                L=16384, cache="i4", weight="f16", rope=False, group=128,
                h2_n=256, h2_m=3, cfg_id=3),
    # LLaVA-v1.5-13B attention layer, bf16, RoPE, ragged lengths, random beta
    4: Workload("llava13b-bf16-rope-ragged", E=5120, H=40, d_h=128, r=2304,
                B=8, L=32768, cache="bf16", weight="bf16", rope=True,
                beta_range=(0.2, 0.8), outlier_frac=0.01, outlier_scale=30.0,
                ragged=(4096, 32768), cfg_id=4),
}

# Same structure as configurations 1..4 at sizes the oracle runs in seconds;
# every one spans several 128-token tiles and ends on a ragged tail.
SHRUNK = {
    1: replace(CONFIGS[1], name="shrunk-fp16-absorbed", E=512, H=4, r=256,
               B=3, L=300),
    2: replace(CONFIGS[2], name="shrunk-bf16-rope", E=512, H=4, r=256, B=2,
               L=290),
    3: replace(CONFIGS[3], name="shrunk-int4-h2", E=512, H=4, r=384, B=3,
               L=270, h2_n=128, h2_m=3),
    4: replace(CONFIGS[4], name="shrunk-bf16-rope-ragged", E=640, H=5,
               r=384, B=3, L=420, ragged=(1, 420)),
}


def rng(w: Workload, stream: str) -> np.random.Generator:
    return np.random.default_rng([w.seed, STREAM[stream]])


def haar_orthogonal(n: int, g: np.random.Generator) -> np.ndarray:
    """n x n Haar-distributed orthogonal matrix (fp64)."""
    a = g.standard_normal((n, n))
    q, rr = np.linalg.qr(a)
    d = np.sign(np.diag(rr))
    d[d == 0] = 1.0
    return q * d[None, :]


def spectrum(E: int, alpha: float = 0.5) -> np.ndarray:
    """Power-law singular values sigma_i = kappa * i**-alpha, ||.||_2^2 = E."""
    i = np.arange(1, E + 1, dtype=np.float64)
    s = i ** (-alpha)
    kappa = math.sqrt(E / float(np.sum(s * s)))
    return kappa * s


def qkv_weights(w: Workload):
    """W_Q, W_K, W_V (E x E, fp32 values) with Haar singular vectors."""
    out = []
    sig = spectrum(w.E)
    for name in ("wq", "wk", "wv"):
        g = rng(w, name)
        u = haar_orthogonal(w.E, g)
        v = haar_orthogonal(w.E, g)
        out.append(((u * sig[None, :]) @ v.T).astype(np.float32))
    return tuple(out)


def outlier_channels(w: Workload) -> np.ndarray:
    g = rng(w, "outliers")
    k = int(round(w.outlier_frac * w.E))
    return np.sort(g.choice(w.E, size=k, replace=False))


def activations(w: Workload, n_tokens: int, stream: str = "x",
                offset_rows: int = 0) -> np.ndarray:
    """X rows (n_tokens x E, fp32): N(0,1) with the seeded outlier channels
    scaled.  ``offset_rows`` skips that many rows of the stream so that one
    long stream can be produced in pieces."""
    g = rng(w, stream)
    if offset_rows:
        g.standard_normal((offset_rows, w.E))
    x = g.standard_normal((n_tokens, w.E))
    x[:, outlier_channels(w)] *= w.outlier_scale
    return x.astype(np.float32)


def sequence_activations(w: Workload, b: int, n_tokens: int) -> np.ndarray:
    """Activations of sequence b (n_tokens x E, fp32), its own sub-stream."""
    g = np.random.default_rng([w.seed, STREAM["x"], b])
    x = g.standard_normal((n_tokens, w.E))
    x[:, outlier_channels(w)] *= w.outlier_scale
    return x.astype(np.float32)


def lengths(w: Workload) -> np.ndarray:
    if w.ragged is None:
        return np.full(w.B, w.L, dtype=np.int32)
    g = rng(w, "lengths")
    lo, hi = w.ragged
    return g.integers(lo, hi + 1, size=w.B).astype(np.int32)


def beta(w: Workload) -> float:
    if w.beta_range is None:
        return w.beta
    g = rng(w, "beta")
    lo, hi = w.beta_range
    return float(g.uniform(lo, hi))


def dct3() -> np.ndarray:
    """Orthonormal 3x3 DCT-II matrix (rows are the basis vectors)."""
    n = 3
    m = np.zeros((n, n))
    for k in range(n):
        a = math.sqrt((1.0 if k == 0 else 2.0) / n)
        for i in range(n):
            m[k, i] = a * math.cos(math.pi * (2 * i + 1) * k / (2 * n))
    return m


def small_orthogonal(m: int) -> np.ndarray:
    """The small Kronecker factor of H2: DCT-II for m = 3, identity otherwise."""
    if m == 3:
        return dct3()
    return np.eye(m)


# ---------------------------------------------------------------------------
# Direct latent inputs (benchmark-scale): random latent rows and up-projection
# rows with a power-law channel profile, drawn without building X or an SVD.
# Channel i of the latent has standard deviation sigma_i**beta and row i of
# each up-projection has scale sigma_i**(1-beta)/sqrt(r), with sigma_i the
# power-law profile above (taken over the first r indices).  A fixed seeded
# 1% of latent channels carries an extra x outlier_scale/4 factor so that the
# per-token range is outlier-dominated, as on the pages' activations.
# ---------------------------------------------------------------------------

def direct_channel_scales(w: Workload):
    sig = spectrum(w.E)[: w.r]
    b = beta(w)
    cs = sig ** b
    ws = sig ** (1.0 - b) / math.sqrt(w.r)
    g = rng(w, "misc")
    k = max(1, int(round(w.outlier_frac * w.r)))
    idx = g.choice(w.r, size=k, replace=False)
    cs = cs.copy()
    cs[idx] *= max(1.0, w.outlier_scale / 4.0)
    return cs, ws


def direct_up_weights_np(w: Workload):
    """W^u_q, W^u_k, W^u_v (r x E each, fp32 values)."""
    _, ws = direct_channel_scales(w)
    g = rng(w, "direct_w")
    out = []
    for _ in range(3):
        out.append((g.standard_normal((w.r, w.E)) * ws[:, None]).astype(np.float32))
    return tuple(out)


def direct_down_weight_np(w: Workload):
    """W^d (E x r, fp32 values) with unit-norm-scale columns times sigma^beta."""
    cs, _ = direct_channel_scales(w)
    g = rng(w, "direct_w")
    g.standard_normal((3, w.r, w.E))  # skip the up-projection draws
    return (g.standard_normal((w.E, w.r)) * (cs / math.sqrt(w.E))[None, :]).astype(np.float32)


def direct_latent_rows_np(w: Workload, b: int, n_tokens: int) -> np.ndarray:
    """Latent rows of sequence b (n_tokens x r, fp32 values)."""
    cs, _ = direct_channel_scales(w)
    g = np.random.default_rng([w.seed, STREAM["direct_c"], b])
    return (g.standard_normal((n_tokens, w.r)) * cs[None, :]).astype(np.float32)


def direct_new_latent_np(w: Workload) -> np.ndarray:
    """Latent of the current token per sequence (B x r, fp32)."""
    cs, _ = direct_channel_scales(w)
    g = rng(w, "direct_cnew")
    return (g.standard_normal((w.B, w.r)) * cs[None, :]).astype(np.float32)


def direct_new_tokens_np(w: Workload) -> np.ndarray:
    """Current-token activations x (B x E, fp32), N(0,1) with outliers."""
    return activations(w, w.B, stream="xnew")
