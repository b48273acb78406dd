"""Split-exponent (beta) search on calibration data, through the library.

QSVD paper notes, 核心创新: the exponent beta that shares the singular values
between the down-projection (W^d = U_r Sigma_r^beta) and the up-projections
(W^u = Sigma_r^(1-beta) V_r^T) is fitted on a calibration set to minimise
sum_d ||Y_d - Y'_d||^2; QSVD digest, Method, Step 3: per layer, on the
self-attention output, with the buffered latent quantised.

One evaluation of the objective runs on the GPU through the C calls:
qsvd_split_factors (the factors for beta), qsvd_prepare_weights (layout, H2
fold), qsvd_prefill_latent three times (the calibration latents rounded to
float32 for Y, quantised into the cache for Y', and the float32 latent of
each sequence's last token, the decode query), and qsvd_decode_attn twice.
Y_d and Y'_d are the decode-step outputs of calibration sequence d (its last
token attending to all its tokens); qsvd_beta_exponents forms sigma^beta and
sigma^(1 - beta) and qsvd_sq_diff_sum adds up the squared differences of the
two B x E outputs in float64 on the device: the host reads one number.

The search: a grid over [0, 1], then a golden-section search (Kiefer, 1953)
between the best grid point's neighbours; the best beta evaluated wins.
"""
from __future__ import annotations

import math
from typing import Dict, Optional, Sequence, Tuple

import numpy as np
import torch

from . import (QSVD_KERNEL_AUTO, make_dims, qsvd_beta_exponents, qsvd_decode_attn, qsvd_prefill_latent,
               qsvd_prepare_weights, qsvd_split_factors, qsvd_sq_diff_sum)

_GOLDEN = (math.sqrt(5.0) - 1.0) / 2.0
_TORCH = {"f16": torch.float16, "bf16": torch.bfloat16}


class BetaObjective:
    """sum_d ||Y_d - Y'_d||^2 as a function of beta for fixed SVD factors and
    calibration sequences.

    u: E x r, s: (r,), vt: r x 3E (the leading singular triplets of
    [W_Q W_K W_V]); x: the calibration activations, sequences concatenated
    (sum(lengths) x E, weight dtype, device); lengths: host ints (each >= 1).
    cache: "i4" or "i8" (group quantiser, ``group`` channels per scale).
    h2_q / h2_m: optional H2 = H_{r/m} (x) Q folded into the factors."""

    def __init__(self, u: torch.Tensor, s: Sequence[float], vt: torch.Tensor, x: torch.Tensor,
                 lengths: Sequence[int], H: int, *, cache: str = "i4", group: int = 128,
                 weight: str = "f16", h2_q=None, h2_m: int = 0, kernel: int = QSVD_KERNEL_AUTO):
        dev = x.device
        E, r = u.shape
        self.s = np.asarray(s, np.float64)
        self.lengths = np.asarray(lengths, np.int64)
        B = len(self.lengths)
        max_len = int(self.lengths.max())
        self.h2_q = h2_q
        kw = dict(weight=weight, group=group, kernel=kernel, h2=False, h2_m=h2_m)
        self.dims_f = make_dims(E, H, E // H, r, B, max_len, cache="f32", **kw)
        self.dims_q = make_dims(E, H, E // H, r, B, max_len, cache=cache, **kw)
        self.dims_last = make_dims(E, H, E // H, r, B, 1, cache="f32", **kw)
        self.u = u.to(dev, torch.float32).contiguous()
        self.vt = vt.to(dev, torch.float32).contiguous()
        self.x = x.contiguous()
        wt = _TORCH[weight]
        self.wd = torch.empty((E, r), dtype=wt, device=dev)
        self.wu = [torch.empty((r, E), dtype=wt, device=dev) for _ in range(3)]
        self.packed = None
        starts = np.concatenate([[0], np.cumsum(self.lengths)[:-1]])
        rows = np.concatenate([b * max_len + np.arange(n) for b, n in enumerate(self.lengths)])
        self.rows = torch.from_numpy(rows.astype(np.int32)).to(dev)
        # the last token of every sequence: its latent is the decode query
        self.x_last = self.x[torch.from_numpy(starts + self.lengths - 1).to(dev)].contiguous()
        self.last_rows = torch.arange(B, dtype=torch.int32, device=dev)
        self.cache_f = torch.empty((B, max_len, r), dtype=torch.float32, device=dev)
        rowb = r // 2 if cache == "i4" else r
        self.cache_q = torch.empty((B, max_len, rowb), dtype=torch.uint8, device=dev)
        self.scales = torch.empty((B, max_len, r // group), dtype=torch.float16, device=dev)
        self.scratch = torch.empty((B, r), dtype=torch.float32, device=dev)
        self.qin = torch.empty((B, r), dtype=torch.float32, device=dev)
        self.len_dev = torch.from_numpy(self.lengths.astype(np.int32)).to(dev)
        self.y = torch.empty((B, E), dtype=torch.float32, device=dev)
        self.yq = torch.empty((B, E), dtype=torch.float32, device=dev)
        self.ws_f = self.ws_q = None
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.sigma = torch.from_numpy(self.s.astype(np.float32)).to(dev)
        self.a = torch.empty(r, dtype=torch.float32, device=dev)
        self.b = torch.empty(r, dtype=torch.float32, device=dev)
        self.obj = torch.zeros(1, dtype=torch.float64, device=dev)
        self.evaluations = 0

    def outputs(self, beta: float) -> Tuple[torch.Tensor, torch.Tensor]:
        """Y (float32 latent rows) and Y' (quantised rows) on the device."""
        qsvd_beta_exponents(self.sigma, beta, self.a, self.b)
        qsvd_split_factors(self.dims_f, self.u, self.vt, self.a, self.b, self.wd, *self.wu)
        self.packed = qsvd_prepare_weights(self.dims_f, self.wd, *self.wu, h2_q=self.h2_q,
                                           packed=self.packed)
        qsvd_prefill_latent(self.dims_f, self.packed, self.x, self.rows, self.cache_f,
                            status=self.status)
        qsvd_prefill_latent(self.dims_q, self.packed, self.x, self.rows, self.cache_q, self.scales,
                            status=self.status)
        qsvd_prefill_latent(self.dims_last, self.packed, self.x_last, self.last_rows, self.scratch,
                            c_out=self.qin, status=self.status)
        self.ws_f = qsvd_decode_attn(self.dims_f, self.packed, self.qin, True, self.cache_f, None,
                                     self.len_dev, self.y, workspace=self.ws_f)
        self.ws_q = qsvd_decode_attn(self.dims_q, self.packed, self.qin, True, self.cache_q,
                                     self.scales, self.len_dev, self.yq, workspace=self.ws_q)
        self.evaluations += 1
        return self.y, self.yq

    def __call__(self, beta: float) -> float:
        y, yq = self.outputs(beta)
        qsvd_sq_diff_sum(y, yq, self.obj)   # on the device, float64
        return float(self.obj.item())

    def status_word(self) -> int:
        return int(self.status.item())


def search_beta(objective, grid: Sequence[float] = tuple(i / 10 for i in range(11)),
                refine: int = 8) -> Tuple[float, float, Dict[float, float]]:
    """Grid, then golden-section refinement between the best grid point's
    neighbours; returns (beta, objective, every evaluation)."""
    seen: Dict[float, float] = {}

    def f(b: float) -> float:
        if b not in seen:
            seen[b] = objective(b)
        return seen[b]

    pts = list(grid)
    i = min(range(len(pts)), key=lambda k: f(pts[k]))
    lo, hi = pts[max(i - 1, 0)], pts[min(i + 1, len(pts) - 1)]
    x1, x2 = hi - _GOLDEN * (hi - lo), lo + _GOLDEN * (hi - lo)
    for _ in range(refine):
        if f(x1) <= f(x2):
            hi, x2 = x2, x1
            x1 = hi - _GOLDEN * (hi - lo)
        else:
            lo, x1 = x1, x2
            x2 = lo + _GOLDEN * (hi - lo)
    best = min(seen, key=lambda b: (seen[b], b))
    return best, seen[best], seen
