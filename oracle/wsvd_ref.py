"""fp64 reference of the per-head (WSVD) latent variant.

Test infrastructure only (see the package docstring).

WSVD paper digest, Method, per-head SVD (§3.1): each head's key (and value)
projection W_{Kh} (E x d_h; the digest writes the head width as H) is
factorised on its own, W_{Kh} = A_{Kh} B_{Kh} with A_{Kh} E x r and B_{Kh}
r x d_h, and each head caches its own latent C_{Kh} = X A_{Kh} (L x r).
Fused kernel (§3.4): keys are rebuilt per tile as C_{Kh,t} B_{Kh}, rotated,
and contracted with q_h; the value factor B_{Vh} is merged into the output
projection.  Key Contributions: the per-head latent traffic per decode step
is L r against L R for a latent of rank R shared by all heads.

Notation here: E = H * d_h, head h owns columns [h d_h, (h+1) d_h) of W_K,
W_V and rows of W_O; r is the per-head rank, R the shared rank.

Readings (the digest leaves them open):
* the singular values are split between the factors as in the joint case,
  A = U_r Sigma_r^beta, B = Sigma_r^(1-beta) V_r^T;
* the query is X W_Q, uncompressed (the digest compresses K and V only);
* every head keeps separate key and value latents.
"""
from __future__ import annotations

import math
from typing import List, Optional, Sequence, Tuple

import numpy as np

from oracle import qsvd_ref as ref


def per_head_factors(w: np.ndarray, H: int, r: int, beta: float = 0.5
                     ) -> List[Tuple[np.ndarray, np.ndarray]]:
    """[(A_h E x r, B_h r x d_h)] for h < H: the rank-r SVD of each head's
    column block of ``w`` (E x E) with the beta split of its singular values."""
    w = np.asarray(w, np.float64)
    E = w.shape[0]
    d_h = E // H
    out = []
    for h in range(H):
        u, s, vt = np.linalg.svd(w[:, h * d_h:(h + 1) * d_h], full_matrices=False)
        out.append((u[:, :r] * (s[:r] ** beta)[None, :], (s[:r] ** (1.0 - beta))[:, None] * vt[:r]))
    return out


def per_head_latents(x: np.ndarray, fac: Sequence[Tuple[np.ndarray, np.ndarray]]) -> np.ndarray:
    """C_h = X A_h for every head: H x L x r."""
    x = np.asarray(x, np.float64)
    return np.stack([x @ a for a, _ in fac])


def decode(ck: Sequence[np.ndarray], cv: Sequence[np.ndarray], lengths, q: np.ndarray,
           fk: Sequence[Tuple[np.ndarray, np.ndarray]], fv: Sequence[Tuple[np.ndarray, np.ndarray]],
           *, rope_base: Optional[float] = None, scale: Optional[float] = None) -> np.ndarray:
    """Decode-step attention over per-head latents.

    ck[b], cv[b]: H x L_b x r key and value latents of sequence b; q: B x E
    query (head h in columns h d_h ..).  Keys K_h = C_{Kh} B_{Kh} and values
    V_h = C_{Vh} B_{Vh} are rebuilt in full, keys (and the query, at position
    len - 1) rotated when rope_base is given.  Output B x E (heads
    concatenated; an empty sequence gives zeros)."""
    H = len(fk)
    d_h = fk[0][1].shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d_h)
    B = len(lengths)
    out = np.zeros((B, H * d_h))
    for b in range(B):
        n = int(lengths[b])
        if n == 0:
            continue
        for h in range(H):
            k = np.asarray(ck[b][h], np.float64)[:n] @ fk[h][1]
            v = np.asarray(cv[b][h], np.float64)[:n] @ fv[h][1]
            qh = np.asarray(q[b, h * d_h:(h + 1) * d_h], np.float64)
            if rope_base is not None:
                k = ref.rope(k, np.arange(n), rope_base)
                qh = ref.rope(qh[None, :], np.array([n - 1]), rope_base)[0]
            out[b, h * d_h:(h + 1) * d_h] = ref.softmax_attention(qh, k, v, scale)
    return out


def decode_absorbed(ck, cv, lengths, q, fk, fv, *, scale: Optional[float] = None) -> np.ndarray:
    """The same without rotary embedding and without rebuilding K or V:
    qt_h = B_{Kh} q_h, scores C_{Kh} qt_h, z_h = p^T C_{Vh}, o_h = z_h B_{Vh}."""
    H = len(fk)
    d_h = fk[0][1].shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d_h)
    B = len(lengths)
    out = np.zeros((B, H * d_h))
    for b in range(B):
        n = int(lengths[b])
        if n == 0:
            continue
        for h in range(H):
            qt = fk[h][1] @ np.asarray(q[b, h * d_h:(h + 1) * d_h], np.float64)
            c_k = np.asarray(ck[b][h], np.float64)[:n]
            s = scale * (c_k @ qt)
            p = np.exp(s - np.max(s))
            z = (p / np.sum(p)) @ np.asarray(cv[b][h], np.float64)[:n]
            out[b, h * d_h:(h + 1) * d_h] = z @ fv[h][1]
    return out


def latent_bytes_per_head(L: int, rank: int, elem_bytes: float) -> float:
    """Latent bytes one head reads per decode step: L x rank elements (the
    digest's eta = L r per head for per-head latents, L R for a shared one)."""
    return float(L) * rank * elem_bytes


def decode_latents(ck, cv, lengths, q, fk, *, scale: Optional[float] = None) -> np.ndarray:
    """z_h = p_h^T C_{Vh} per sequence and head (B x H x r), scores from the
    absorbed query (no rotary embedding)."""
    H = len(fk)
    d_h = fk[0][1].shape[1]
    r = fk[0][1].shape[0]
    if scale is None:
        scale = 1.0 / math.sqrt(d_h)
    B = len(lengths)
    z = np.zeros((B, H, r))
    for b in range(B):
        n = int(lengths[b])
        if n == 0:
            continue
        for h in range(H):
            qt = fk[h][1] @ np.asarray(q[b, h * d_h:(h + 1) * d_h], np.float64)
            s = scale * (np.asarray(ck[b][h], np.float64)[:n] @ qt)
            p = np.exp(s - np.max(s))
            z[b, h] = (p / np.sum(p)) @ np.asarray(cv[b][h], np.float64)[:n]
    return z


def fold_values(fv: Sequence[Tuple[np.ndarray, np.ndarray]], wo: np.ndarray) -> np.ndarray:
    """Fused kernel (§3.4): B_{Vh} merged into the output projection,
    F_h = B_{Vh} W_{O,h} (r x E, W_{O,h} the rows h d_h .. of W_O), stacked
    by head (H r x E)."""
    wo = np.asarray(wo, np.float64)
    d_h = fv[0][1].shape[1]
    return np.concatenate([b @ wo[h * d_h:(h + 1) * d_h] for h, (_, b) in enumerate(fv)])


def out_proj_weight_elems(E: int, H: int, r: int, folded: bool) -> int:
    """Weight elements the output stage reads per step: H r E folded, or the
    per-head value factors plus W_O (H r d_h + E^2) unfolded."""
    return H * r * E if folded else H * r * (E // H) + E * E
