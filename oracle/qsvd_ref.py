"""fp64 reference of joint-QKV SVD compression and latent decode attention.

Test infrastructure only (see the package docstring).

Notation: E = H * d_h model width, r the retained rank, L tokens per
sequence.  Head h owns columns [h*d_h, (h+1)*d_h) of every E-wide projection
(standard multi-head split).  Latent rows are tokens: C is L x r.
"""
from __future__ import annotations

import math
from typing import Optional, Sequence

import numpy as np


# --------------------------------------------------------------------------
# Offline compression
# --------------------------------------------------------------------------

def joint_svd(wq: np.ndarray, wk: np.ndarray, wv: np.ndarray):
    """SVD of the concatenation [W_Q W_K W_V] (E x 3E).

    QSVD paper notes, 关键设计 (QKV joint SVD); QSVD digest, Method, Step 1:
    the three E x E projections are concatenated along the output dimension
    and decomposed once.  Returns (U, sigma, V^T) with U E x E, sigma (E,),
    V^T E x 3E (LAPACK, float64)."""
    w = np.concatenate([np.asarray(wq, np.float64), np.asarray(wk, np.float64),
                        np.asarray(wv, np.float64)], axis=1)
    u, s, vt = np.linalg.svd(w, full_matrices=False)
    return u, s, vt


def factors(u: np.ndarray, s: np.ndarray, vt: np.ndarray, r: int, beta: float):
    """Rank-r factors with the beta split of Sigma.

    QSVD paper notes, 关键设计 (SVD-compatible quantisation): the buffered
    latent is X W^d_r Sigma_r^beta; QSVD digest, Method, Step 3: beta decides
    how the singular values are shared between the down- and up-projection.
    Reading (the pages leave it open): the up-projection carries the rest,
    Sigma_r^(1-beta), so that W^d W^u equals the truncated SVD.

    Returns W^d (E x r) and W^u_q, W^u_k, W^u_v (each r x E)."""
    E = u.shape[0]
    sr = s[:r]
    wd = u[:, :r] * (sr ** beta)[None, :]
    wu = (sr ** (1.0 - beta))[:, None] * vt[:r, :]
    return wd, wu[:, :E], wu[:, E:2 * E], wu[:, 2 * E:3 * E]


def truncation_residual(wq, wk, wv, wd, wuq, wuk, wuv) -> float:
    """||[W_Q W_K W_V] - W^d [W^u_q W^u_k W^u_v]||_F^2, formed explicitly."""
    w = np.concatenate([wq, wk, wv], axis=1).astype(np.float64)
    approx = wd @ np.concatenate([wuq, wuk, wuv], axis=1)
    return float(np.sum((w - approx) ** 2))


def param_counts(E: int, r: int, L: int) -> dict:
    """Parameter and cache sizes (elements), joint vs per-matrix SVD.

    QSVD paper notes, 关键设计; QSVD digest, Problem and Key Contributions:
    one shared E x r down-projection plus three r x E up-projections, and one
    L x r latent per sequence, against a down/up pair per matrix and separate
    key and value latents."""
    joint_params = E * r + 3 * (r * E)
    per_matrix_params = 3 * (E * r + r * E)
    return {
        "joint_params": joint_params,
        "per_matrix_params": per_matrix_params,
        "joint_cache": r * L,
        "per_matrix_cache": 2 * r * L,
        "dense_params": 3 * E * E,
        "dense_cache": 2 * E * L,
    }


def cache_ratio(E: int, r: int) -> float:
    """Latent cache size relative to an uncompressed K+V cache: rL / (2EL)."""
    return r / (2.0 * E)


def compression_active(E: int, r: int) -> bool:
    """Joint factors hold fewer weights than the dense Q, K, V projections
    (4rE < 3E^2, i.e. r < 0.75 E; QSVD digest, Method, Step 1)."""
    return 4 * r * E < 3 * E * E


# --------------------------------------------------------------------------
# Rotation H2 = H_n (x) Q_m
# --------------------------------------------------------------------------

def hadamard(n: int) -> np.ndarray:
    """Normalised Sylvester Hadamard matrix of order n (a power of two),
    entry (i, j) = (-1)^popcount(i & j) / sqrt(n)."""
    if n < 1 or (n & (n - 1)):
        raise ValueError("Hadamard order must be a power of two")
    i = np.arange(n)
    bits = np.bitwise_and(i[:, None], i[None, :])
    parity = np.zeros_like(bits)
    b = bits.copy()
    while np.any(b):
        parity ^= (b & 1)
        b >>= 1
    return np.where(parity == 1, -1.0, 1.0) / math.sqrt(n)


def h2_matrix(n: int, q: np.ndarray) -> np.ndarray:
    """H2 = H_n (x) Q (r x r with r = n * m).  QSVD paper notes, 关键设计:
    an orthogonal H2 placed between the down- and up-projection, so that
    Y = (X H1^T)(H1 W^d H2^T)(H2 W^u)."""
    return np.kron(hadamard(n), np.asarray(q, np.float64))


def rotate_factors(wd, wuq, wuk, wuv, h2: np.ndarray):
    """Fold H2 into the factors: W^d <- W^d H2^T, W^u_* <- H2 W^u_*."""
    return wd @ h2.T, h2 @ wuq, h2 @ wuk, h2 @ wuv


# --------------------------------------------------------------------------
# Latent cache and decode attention
# --------------------------------------------------------------------------

def latent(x: np.ndarray, wd: np.ndarray) -> np.ndarray:
    """C = X W^d (rows are tokens).  QSVD paper notes, 关键设计; QSVD digest,
    Method, Step 1 (the buffered intermediate)."""
    return np.asarray(x, np.float64) @ np.asarray(wd, np.float64)


def rope_angles(positions: np.ndarray, d_h: int, base: float) -> np.ndarray:
    """theta_i * p for i < d_h/2, theta_i = base^(-2i/d_h)."""
    i = np.arange(d_h // 2, dtype=np.float64)
    theta = base ** (-2.0 * i / d_h)
    return np.asarray(positions, np.float64)[:, None] * theta[None, :]


def rope(v: np.ndarray, positions: np.ndarray, base: float) -> np.ndarray:
    """Rotary embedding on the last axis (rotate-half pairing (i, i + d/2)).

    The WSVD digest (Method, fused kernel 3.4) applies rotary embedding to the
    reconstructed keys; the pairing and base are not stated there -- the
    LLaMA/LLaVA convention is taken.  v: (n, d_h), positions: (n,)."""
    v = np.asarray(v, np.float64)
    d = v.shape[-1]
    half = d // 2
    ang = rope_angles(positions, d, base)
    c, s = np.cos(ang), np.sin(ang)
    a, b = v[..., :half], v[..., half:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


def softmax_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray,
                      scale: float) -> np.ndarray:
    """Single-query attention: softmax(scale * k q) over rows of k, then p v."""
    s = scale * (k @ q)
    if s.size == 0:
        return np.zeros(v.shape[1])
    s = s - np.max(s)
    p = np.exp(s)
    p /= np.sum(p)
    return p @ v


def decode_materialized(caches: Sequence[np.ndarray], lengths, qin: np.ndarray,
                        wuq, wuk, wuv, H: int, *, qin_is_latent: bool = True,
                        rope_base: Optional[float] = None,
                        scale: Optional[float] = None) -> np.ndarray:
    """Decode-step multi-head attention with K and V rebuilt from the latent.

    QSVD digest, Method, Step 1: keys and values are recomputed on the fly as
    C W^u_k and C W^u_v.  Here they are materialised in full (L x E) and
    textbook attention runs per head.

    caches[b]: L_b x r latent rows of sequence b (at least lengths[b] rows).
    qin: B x r latent of the current token (q = c_new W^u_q) or, with
    qin_is_latent=False, the B x E query itself.
    rope_base: None for no rotary embedding; otherwise keys at positions
    0..len-1 and the query at position len-1 are rotated.
    Output: B x E (heads concatenated)."""
    wuq = np.asarray(wuq, np.float64)
    wuk = np.asarray(wuk, np.float64)
    wuv = np.asarray(wuv, np.float64)
    E = wuk.shape[1]
    d_h = E // H
    if scale is None:
        scale = 1.0 / math.sqrt(d_h)
    B = len(lengths)
    out = np.zeros((B, E))
    for b in range(B):
        n = int(lengths[b])
        c = np.asarray(caches[b], np.float64)[:n]
        qb = np.asarray(qin[b], np.float64)
        q = qb @ wuq if qin_is_latent else qb
        k = c @ wuk
        v = c @ wuv
        for h in range(H):
            cols = slice(h * d_h, (h + 1) * d_h)
            qh, kh = q[cols], k[:, cols]
            if rope_base is not None and n > 0:
                kh = rope(kh, np.arange(n), rope_base)
                qh = rope(qh[None, :], np.array([n - 1]), rope_base)[0]
            out[b, cols] = softmax_attention(qh, kh, v[:, cols], scale)
    return out


def decode_absorbed(caches: Sequence[np.ndarray], lengths, qin: np.ndarray,
                    wuq, wuk, wuv, H: int, *, qin_is_latent: bool = True,
                    scale: Optional[float] = None) -> np.ndarray:
    """Same attention without rebuilding K or V (no rotary embedding).

    The query is absorbed into the latent space, qt_h = W^u_{k,h} q_h, so the
    scores are C qt_h; the value side is accumulated in latent space,
    z_h = p^T C, and up-projected once, o_h = z_h W^u_{v,h}."""
    wuq = np.asarray(wuq, np.float64)
    wuk = np.asarray(wuk, np.float64)
    wuv = np.asarray(wuv, np.float64)
    E = wuk.shape[1]
    d_h = E // H
    if scale is None:
        scale = 1.0 / math.sqrt(d_h)
    B = len(lengths)
    out = np.zeros((B, E))
    for b in range(B):
        n = int(lengths[b])
        c = np.asarray(caches[b], np.float64)[:n]
        qb = np.asarray(qin[b], np.float64)
        q = qb @ wuq if qin_is_latent else qb
        for h in range(H):
            cols = slice(h * d_h, (h + 1) * d_h)
            qt = wuk[:, cols] @ q[cols]
            if n == 0:
                continue
            s = scale * (c @ qt)
            s -= np.max(s)
            p = np.exp(s)
            p /= np.sum(p)
            z = p @ c
            out[b, cols] = z @ wuv[:, cols]
    return out


def attention_uncompressed(xs: Sequence[np.ndarray], lengths, x_query: np.ndarray,
                           wq, wk, wv, H: int, *, rope_base: Optional[float] = None,
                           scale: Optional[float] = None) -> np.ndarray:
    """Dense multi-head attention on X W_Q, X W_K, X W_V (no compression).

    xs[b]: L_b x E activations of sequence b; x_query: B x E activation of the
    current token.  Written independently of the latent routines above."""
    wq = np.asarray(wq, np.float64)
    wk = np.asarray(wk, np.float64)
    wv = np.asarray(wv, np.float64)
    E = wq.shape[0]
    d_h = E // H
    if scale is None:
        scale = 1.0 / math.sqrt(d_h)
    out = np.zeros((len(lengths), E))
    for b in range(len(lengths)):
        n = int(lengths[b])
        x = np.asarray(xs[b], np.float64)[:n]
        q = np.asarray(x_query[b], np.float64) @ wq
        kk = x @ wk
        vv = x @ wv
        for h in range(H):
            lo, hi = h * d_h, (h + 1) * d_h
            qh, kh = q[lo:hi], kk[:, lo:hi]
            if rope_base is not None and n > 0:
                kh = rope(kh, np.arange(n), rope_base)
                qh = rope(qh[None, :], np.array([n - 1]), rope_base)[0]
            logits = scale * (kh @ qh)
            m = np.max(logits)
            e = np.exp(logits - m)
            out[b, lo:hi] = (e / e.sum()) @ vv[:, lo:hi]
    return out


# --------------------------------------------------------------------------
# Output projection (the layer's W_O after attention)
# --------------------------------------------------------------------------

def output_projection(o: np.ndarray, wo: np.ndarray) -> np.ndarray:
    """y = o W_O: the attention output (B x E, heads concatenated) times the
    layer's output projection (E x E; row h*d_h + i multiplies channel i of
    head h)."""
    return np.asarray(o, np.float64) @ np.asarray(wo, np.float64)


def fold_value_output(wuv: np.ndarray, wo: np.ndarray, H: int) -> np.ndarray:
    """Per-head merge of the value up-projection into the output projection.

    WSVD digest, Method, fused kernel (§3.4): the value factor of each head
    is fused into the output projection so that V is never rebuilt.  With a
    shared latent the value factor of head h is W^u_{v,h} (the d_h columns of
    W^u_v that belong to h, r x d_h) and the matching slice of W_O is its rows
    h*d_h .. h*d_h + d_h - 1 (d_h x E).  Returns F stacked by head: rows
    h*r .. h*r + r - 1 hold F_h = W^u_{v,h} W_{O,h} (H*r x E)."""
    wuv = np.asarray(wuv, np.float64)
    wo = np.asarray(wo, np.float64)
    r, E = wuv.shape
    d_h = E // H
    f = np.zeros((H * r, wo.shape[1]))
    for h in range(H):
        cols = slice(h * d_h, (h + 1) * d_h)
        f[h * r:(h + 1) * r] = wuv[:, cols] @ wo[cols]
    return f


def decode_absorbed_latents(caches: Sequence[np.ndarray], lengths, qin: np.ndarray,
                            wuq, wuk, H: int, *, qin_is_latent: bool = True,
                            rope_base: Optional[float] = None,
                            scale: Optional[float] = None) -> np.ndarray:
    """Per-head attention-weighted latent z_h = p_h^T C (B x H x r): the
    decode before any value projection (zero for an empty sequence).  The
    scores are C qt_h with qt_h = W^u_{k,h} q_h, or, with rope_base, the
    rotated rebuilt keys R(t) (C W^u_{k,h})_t against the rotated query."""
    wuq = np.asarray(wuq, np.float64)
    wuk = np.asarray(wuk, np.float64)
    E = wuk.shape[1]
    r = wuk.shape[0]
    d_h = E // H
    if scale is None:
        scale = 1.0 / math.sqrt(d_h)
    B = len(lengths)
    z = np.zeros((B, H, r))
    for b in range(B):
        n = int(lengths[b])
        if n == 0:
            continue
        c = np.asarray(caches[b], np.float64)[:n]
        qb = np.asarray(qin[b], np.float64)
        q = qb @ wuq if qin_is_latent else qb
        for h in range(H):
            cols = slice(h * d_h, (h + 1) * d_h)
            if rope_base is None:
                s = scale * (c @ (wuk[:, cols] @ q[cols]))
            else:
                kh = rope(c @ wuk[:, cols], np.arange(n), rope_base)
                qh = rope(q[cols][None, :], np.array([n - 1]), rope_base)[0]
                s = scale * (kh @ qh)
            p = np.exp(s - np.max(s))
            z[b, h] = (p / np.sum(p)) @ c
    return z


def decode_folded(z: np.ndarray, f: np.ndarray) -> np.ndarray:
    """y_b = sum_h z_{b,h} F_h: the projected layer output straight from the
    per-head latents (B x E_out)."""
    z = np.asarray(z, np.float64)
    B, H, r = z.shape
    return z.reshape(B, H * r) @ np.asarray(f, np.float64)


# --------------------------------------------------------------------------
# Prefill attention (all prompt tokens at once, causal)
# --------------------------------------------------------------------------

def prefill_attention(c: np.ndarray, wuq, wuk, wuv, H: int, *, rope_base: Optional[float] = None,
                      scale: Optional[float] = None) -> np.ndarray:
    """Causal self-attention over one prompt whose latent rows are ``c``
    (L x r): Q = C W^u_q, K = C W^u_k, V = C W^u_v rebuilt in full (QSVD
    digest, Method, Step 1), token t attends to tokens 0..t; with rope_base
    every query and key is rotated by its own position.  Output L x E
    (heads concatenated)."""
    c = np.asarray(c, np.float64)
    wuq = np.asarray(wuq, np.float64)
    wuk = np.asarray(wuk, np.float64)
    wuv = np.asarray(wuv, np.float64)
    L = c.shape[0]
    E = wuk.shape[1]
    d_h = E // H
    if scale is None:
        scale = 1.0 / math.sqrt(d_h)
    q, k, v = c @ wuq, c @ wuk, c @ wuv
    out = np.zeros((L, E))
    pos = np.arange(L)
    for h in range(H):
        cols = slice(h * d_h, (h + 1) * d_h)
        qh, kh = q[:, cols], k[:, cols]
        if rope_base is not None:
            qh, kh = rope(qh, pos, rope_base), rope(kh, pos, rope_base)
        logits = scale * (qh @ kh.T)
        logits[np.triu_indices(L, 1)] = -np.inf
        logits -= logits.max(axis=1, keepdims=True)
        p = np.exp(logits)
        p /= p.sum(axis=1, keepdims=True)
        out[:, cols] = p @ v[:, cols]
    return out
