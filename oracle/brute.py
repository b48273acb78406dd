"""Pure-Python loop attention for tiny inputs (no NumPy linear algebra).

Test infrastructure only.  Used to pin ``qsvd_ref.decode_materialized`` and
``qsvd_ref.decode_absorbed`` against the plain definition of decode-step
multi-head attention over keys/values rebuilt from the latent (QSVD digest,
Method, Step 1), one scalar at a time.
"""
from __future__ import annotations

import math


def matvec_row(row, mat, col0, ncols):
    """sum_j row[j] * mat[j][col0 + i] for i < ncols."""
    out = [0.0] * ncols
    for j, rj in enumerate(row):
        mj = mat[j]
        for i in range(ncols):
            out[i] += rj * mj[col0 + i]
    return out


def rotate_pairs(vec, pos, base):
    """Rotary embedding of one head vector, pairs (i, i + d/2), angle
    pos * base^(-2i/d), written with scalar cos/sin."""
    d = len(vec)
    half = d // 2
    out = list(vec)
    for i in range(half):
        ang = pos * base ** (-2.0 * i / d)
        c, s = math.cos(ang), math.sin(ang)
        out[i] = vec[i] * c - vec[i + half] * s
        out[i + half] = vec[i + half] * c + vec[i] * s
    return out


def decode_loops(cache, n, qin, wuq, wuk, wuv, H, scale=None, rope_base=None):
    """One sequence: cache rows (lists), n tokens, qin latent (list of r).
    With rope_base, key t sits at position t and the query at n - 1."""
    r = len(qin)
    E = len(wuq[0])
    d_h = E // H
    if scale is None:
        scale = 1.0 / math.sqrt(d_h)
    q = matvec_row(qin, wuq, 0, E)
    out = [0.0] * E
    for h in range(H):
        c0 = h * d_h
        keys = [matvec_row(cache[t], wuk, c0, d_h) for t in range(n)]
        vals = [matvec_row(cache[t], wuv, c0, d_h) for t in range(n)]
        qh = q[c0:c0 + d_h]
        if rope_base is not None:
            keys = [rotate_pairs(keys[t], t, rope_base) for t in range(n)]
            qh = rotate_pairs(qh, n - 1, rope_base)
        logits = []
        for t in range(n):
            acc = 0.0
            for i in range(d_h):
                acc += qh[i] * keys[t][i]
            logits.append(scale * acc)
        m = max(logits)
        w = [math.exp(x - m) for x in logits]
        tot = sum(w)
        for i in range(d_h):
            acc = 0.0
            for t in range(n):
                acc += w[t] * vals[t][i]
            out[c0 + i] = acc / tot
    assert len(cache[0]) == r
    return out
