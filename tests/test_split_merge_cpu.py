"""Host replay of the split kernels' online softmax and the merge
(split_tc.cu softmax warps, combine.cu k_merge), float64, no GPU.

Per split and head the tensor-core kernel keeps a reference max m (log2
domain) and rescales l and Z only when some score of a tile exceeds m by
more than 2^8 (any head of the warp group triggers it for the group;
heads whose max did not grow get a factor 1); P = 2^(s - m) is then at
most 2^8.  Splits report (m, l, z); the merge weighs split s by
2^(m_s - M) with M the largest m, and divides by the weighted sum of l.
These tests restate those rules and check that the result is the one-pass
softmax average, that P never exceeds 2^8, and that rows past a length
(score -inf) contribute nothing.  The oracle itself takes one softmax over
all tokens, so this is the pin for the split-merge algebra.
"""
import os
import re

import numpy as np
import pytest

RESCALE = 8.0
TILE = 128


def split_partials(s, c, tb, te):
    """One split over tiles [tb, te) of one sequence: scores s [T][H]
    (-inf past the length), latent rows c [T][r].  Returns m, l, z, max P."""
    H = s.shape[1]
    m = np.full(H, -np.inf)
    l = np.zeros(H)
    z = np.zeros((H, c.shape[1]))
    pmax = 0.0
    for i, t0 in enumerate(range(tb * TILE, te * TILE, TILE)):
        st, ct = s[t0:t0 + TILE], c[t0:t0 + TILE]
        first = i == 0
        need = first or bool(np.any(st > m + RESCALE))
        if need:
            mt = st.max(axis=0)
            mn = np.maximum(m, mt) if not first else mt
            with np.errstate(invalid="ignore"):
                a = np.exp2(m - mn) if not first else np.zeros(H)
            a = np.where(np.isfinite(a), a, 0.0)
            l = l * a
            z = z * a[:, None]
            m = mn
        with np.errstate(invalid="ignore"):
            p = np.exp2(st - m)                      # [tile][H]
        p = np.where(np.isfinite(st), p, 0.0)
        pmax = max(pmax, float(p.max(initial=0.0)))
        l = l + p.sum(axis=0)
        z = z + p.T @ ct
    return m, l, z, pmax


def merge(parts):
    """k_merge: M = max m_s; w_s = 2^(m_s - M) / sum_s 2^(m_s - M) l_s."""
    ms = np.stack([p[0] for p in parts])
    M = ms.max(axis=0)
    w = np.exp2(ms - M)
    L = (w * np.stack([p[1] for p in parts])).sum(axis=0)
    z = sum(w[k][:, None] * parts[k][2] for k in range(len(parts)))
    return z / L[:, None]


@pytest.mark.parametrize("seed,n,splits", [(0, 1000, 1), (1, 1000, 3), (2, 4096, 7),
                                           (3, 300, 2), (4, 129, 2), (5, 8192, 13)])
def test_online_softmax_and_merge_equal_the_one_pass_softmax(seed, n, splits):
    g = np.random.default_rng(seed)
    H, r = 6, 40
    T = -(-n // TILE) * TILE
    # scores with drifts and jumps (a new maximum far above the old one
    # late in the sequence), in log2 units
    s = g.standard_normal((T, H)) * 3 + np.linspace(0, 30, T)[:, None] * g.uniform(-1, 1, H)
    s[g.integers(0, n, 5)] += 40
    s[n:] = -np.inf                                   # rows past the length
    c = g.standard_normal((T, r))
    c[n:] = 1e30                                      # would poison a sum if P were not 0 there
    tiles = T // TILE
    bounds = [k * tiles // splits for k in range(splits + 1)]
    parts = [split_partials(s, c, bounds[k], bounds[k + 1]) for k in range(splits)
             if bounds[k + 1] > bounds[k]]
    assert max(p[3] for p in parts) <= 2.0 ** RESCALE
    got = merge(parts)
    sv = s[:n]
    p = np.exp2(sv - sv.max(axis=0))
    want = (p.T @ c[:n]) / p.sum(axis=0)[:, None]
    assert np.max(np.abs(got - want)) <= 1e-12 * np.max(np.abs(want))


def test_the_replay_uses_the_kernels_rules():
    """The threshold and the update rules above are the sources'."""
    csrc = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "rank_joint_qkv_b200",
                        "csrc")
    sp = open(os.path.join(csrc, "split_tc.cu")).read()
    cb = open(os.path.join(csrc, "combine.cu")).read()
    assert re.search(r"constexpr float kRescaleLog2 = 8\.f;", sp)
    assert "need |= sv[h] > s.m_run[hb + h] + kRescaleLog2;" in sp
    assert "const float mn = fmaxf(mo, mt);" in sp and "const float a = exp2f(mo - mn);" in sp
    assert "s.l_run[h] = first ? 0.f : s.l_run[h] * a;" in sp
    assert "const float p = valid ? exp2f(sv[h] - mr[h]) : 0.f;" in sp
    assert "w = exp2f(__ldcg(pm + (size_t(c) + b) * H + h) - M);" in cb
    assert "L += w * __ldcg(pl + (size_t(c) + b) * H + h);" in cb
    assert "const float invL = L > 0.f ? 1.f / L : 0.f;" in cb
