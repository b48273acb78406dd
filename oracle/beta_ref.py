"""fp64 reference of the beta search on calibration data.

Test infrastructure only (see the package docstring).

QSVD paper notes, 核心创新: beta, the exponent that splits the singular
values between the down- and the up-projection, is fitted on a calibration
set so that the quantised model's outputs stay close to the unquantised
ones, min_beta sum_d ||Y_d - Y'_d||^2.  QSVD digest, Method, Step 3: one beta
per layer, the error measured on the self-attention output with the buffered
latent C_qkv quantised.

Readings (the pages name the objective, not its parts):

* Y_d is the decode-step attention output of calibration sequence d (its
  last token attends to all its tokens), computed from the float32 latent
  rows; Y'_d is the same output with the rows quantised by the cache's
  group quantiser.  The query is the float32 latent of the last token in
  both (the decode path's query is never quantised).
* The factors for a given beta are W^d = U_r Sigma_r^beta and
  W^u = Sigma_r^(1-beta) V_r^T (``qsvd_ref.factors``), rounded to the weight
  type the decode path stores; with H2 those stored factors are rotated and
  rounded again.
* The search is a grid over [0, 1] followed by a golden-section search
  (Kiefer, 1953) in the bracket formed by the best grid point's neighbours;
  it returns the best beta evaluated.
"""
from __future__ import annotations

import math
from typing import Callable, Dict, Optional, Sequence, Tuple

import numpy as np

from oracle import inputs as oi
from oracle import quant_ref as qr
from oracle import qsvd_ref as ref

GOLDEN = (math.sqrt(5.0) - 1.0) / 2.0


def _rounded(m: np.ndarray, weight: str) -> np.ndarray:
    return oi.from_device_dtype(oi.to_device_dtype(m, weight), weight)


def beta_weights(u: np.ndarray, s: np.ndarray, vt: np.ndarray, r: int, beta: float,
                 weight: str, h2: Optional[np.ndarray] = None):
    """Factors for ``beta`` as the decode path stores them (float64 values of
    the rounded weights): W^d (E x r), W^u_q, W^u_k, W^u_v (r x E).  The
    factors are rounded to the weight type; H2, when given, rotates those
    rounded factors and the result is rounded again (the rotation is a
    layout step applied to stored weights)."""
    f = tuple(_rounded(m, weight) for m in ref.factors(u, s, vt, r, beta))
    if h2 is not None:
        f = tuple(_rounded(m, weight) for m in ref.rotate_factors(*f, h2))
    return f


def calibration_objective(u, s, vt, r: int, beta: float, xs: Sequence[np.ndarray], lengths,
                          H: int, *, bits: int, group: int, weight: str = "f16",
                          h2: Optional[np.ndarray] = None) -> float:
    """sum_d ||Y_d - Y'_d||^2 over the calibration sequences ``xs`` (each
    at least lengths[d] x E activations, float values of the weight type)."""
    wd, wuq, wuk, wuv = beta_weights(u, s, vt, r, beta, weight, h2)
    ref_rows, quant_rows = [], []
    cnew = np.zeros((len(lengths), r), np.float32)
    for d, x in enumerate(xs):
        n = int(lengths[d])
        c32 = ref.latent(np.asarray(x, np.float64)[:n], wd).astype(np.float32)
        codes, scales, _ = qr.quantize(c32, bits, group)
        ref_rows.append(c32.astype(np.float64))
        quant_rows.append(qr.dequantize(codes, scales, group).astype(np.float64))
        cnew[d] = c32[n - 1]
    q = cnew.astype(np.float64)
    y = ref.decode_absorbed(ref_rows, lengths, q, wuq, wuk, wuv, H)
    yq = ref.decode_absorbed(quant_rows, lengths, q, wuq, wuk, wuv, H)
    return float(np.sum((y - yq) ** 2))


def search(objective: Callable[[float], float], grid: Sequence[float], refine: int
           ) -> Tuple[float, float, Dict[float, float]]:
    """Grid, then golden-section refinement between the best grid point's
    neighbours.  Returns (beta, objective, every evaluation)."""
    evals: Dict[float, float] = {}

    def f(b: float) -> float:
        if b not in evals:
            evals[b] = objective(b)
        return evals[b]

    grid = list(grid)
    vals = [f(b) for b in grid]
    i = int(np.argmin(vals))
    lo, hi = grid[max(i - 1, 0)], grid[min(i + 1, len(grid) - 1)]
    x1, x2 = hi - GOLDEN * (hi - lo), lo + GOLDEN * (hi - lo)
    for _ in range(refine):
        if f(x1) <= f(x2):
            hi, x2 = x2, x1
            x1 = hi - GOLDEN * (hi - lo)
        else:
            lo, x1 = x1, x2
            x2 = lo + GOLDEN * (hi - lo)
    best = min(evals, key=lambda b: (evals[b], b))
    return best, evals[best], evals
