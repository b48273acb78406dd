"""Pins of the per-head (WSVD) latent oracle (``oracle.wsvd_ref``), no GPU.

* Full per-head rank: the factorisation is exact, so the decode equals the
  dense multi-head attention written independently in ``qsvd_ref``, with and
  without rotary embedding.
* Eckart-Young per head: the truncation residual of each head's block is the
  sum of its dropped squared singular values (from a different LAPACK route).
* Absorbing the query and accumulating values in latent space changes only
  the order of the arithmetic.
* Folding B_{Vh} into W_O gives the projected attention; the folded weights
  are smaller than B_V plus W_O exactly when H r E < H r d_h + E^2.
"""
import math

import numpy as np
import pytest
import scipy.linalg

import synthetic
from oracle import qsvd_ref as ref
from oracle import wsvd_ref as wr


def _case(r, L=40, B=3, rope=False):
    w = synthetic.replace(synthetic.SHRUNK[1], E=256, H=4, r=r, B=B, L=L)
    wq, wk, wv = synthetic.qkv_weights(w)
    lens = np.array([L, L // 2 + 1, 1][:B], np.int32)
    xs = [synthetic.sequence_activations(w, b, L).astype(np.float64) for b in range(B)]
    xq = np.stack([xs[b][lens[b] - 1] for b in range(B)])
    fk = wr.per_head_factors(wk, w.H, r)
    fv = wr.per_head_factors(wv, w.H, r)
    ck = [wr.per_head_latents(x, fk) for x in xs]
    cv = [wr.per_head_latents(x, fv) for x in xs]
    return w, (wq, wk, wv), xs, xq, lens, fk, fv, ck, cv


@pytest.mark.parametrize("rope", [False, True])
def test_full_rank_equals_dense_attention(rope):
    w, (wq, wk, wv), xs, xq, lens, fk, fv, ck, cv = _case(r=64)   # d_h = 64
    rb = 10000.0 if rope else None
    got = wr.decode(ck, cv, lens, xq @ wq.astype(np.float64), fk, fv, rope_base=rb)
    want = ref.attention_uncompressed(xs, lens, xq, wq, wk, wv, w.H, rope_base=rb)
    assert np.max(np.abs(got - want)) <= 1e-10 * np.max(np.abs(want))


@pytest.mark.parametrize("r", [8, 24, 63])
def test_eckart_young_per_head(r):
    w = synthetic.replace(synthetic.SHRUNK[1], E=256, H=4)
    _, wk, _ = synthetic.qkv_weights(w)
    d_h = w.E // w.H
    for h, (a, b) in enumerate(wr.per_head_factors(wk, w.H, r, beta=0.3)):
        blk = wk[:, h * d_h:(h + 1) * d_h].astype(np.float64)
        sv = scipy.linalg.svd(blk, compute_uv=False, lapack_driver="gesvd")
        resid = np.sum((blk - a @ b) ** 2)
        assert abs(resid - np.sum(sv[r:] ** 2)) <= 1e-9 * np.sum(blk ** 2)


def test_absorbed_equals_materialised():
    w, (wq, _, _), xs, xq, lens, fk, fv, ck, cv = _case(r=24)
    q = xq @ wq.astype(np.float64)
    got = wr.decode_absorbed(ck, cv, lens, q, fk, fv)
    want = wr.decode(ck, cv, lens, q, fk, fv)
    assert np.max(np.abs(got - want)) <= 1e-11 * np.max(np.abs(want))


def test_fold_values_into_output_projection():
    w, (wq, _, _), xs, xq, lens, fk, fv, ck, cv = _case(r=24)
    q = xq @ wq.astype(np.float64)
    wo = np.random.default_rng(3).standard_normal((w.E, w.E)) / math.sqrt(w.E)
    want = ref.output_projection(wr.decode(ck, cv, lens, q, fk, fv), wo)
    z = wr.decode_latents(ck, cv, lens, q, fk)
    got = z.reshape(len(lens), -1) @ wr.fold_values(fv, wo)
    assert np.max(np.abs(got - want)) <= 1e-11 * np.max(np.abs(want))


def test_fold_pays_below_model_width():
    E, H = 4096, 32
    for r in (16, 64, 120):                       # H r < E: folding reads fewer weights
        assert wr.out_proj_weight_elems(E, H, r, True) < wr.out_proj_weight_elems(E, H, r, False)
    # a shared latent of rank 1536 read by all 32 heads: folding reads 8.7x more
    ratio = wr.out_proj_weight_elems(E, H, 1536, True) / (1536 * E + E * E)
    assert 8.6 < ratio < 8.8


def test_per_head_traffic_ratio():
    """Key Contributions: per head and step, a per-head latent moves L r
    elements where a shared one moves L R, a ratio r / R.  LLaVA-7B shapes:
    a shared latent of rank 1536 read for each of 32 heads against per-head
    key and value latents of rank 64."""
    L = 8192
    assert wr.latent_bytes_per_head(L, 64, 2) / wr.latent_bytes_per_head(L, 1536, 2) == 64 / 1536
    shared_reloaded = 32 * wr.latent_bytes_per_head(L, 1536, 2)
    per_head_kv = 32 * 2 * wr.latent_bytes_per_head(L, 64, 2)
    assert shared_reloaded == 805306368 and per_head_kv == 67108864
