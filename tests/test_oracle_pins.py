"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test would fail on a plausible slip in the oracle (a dropped Sigma
factor, a wrong head split or transposed factor, a missing scale, a wrong
rotation pairing, a rounding mode): see the comment on each.
"""
import math
import os
import struct

import numpy as np
import pytest
import scipy.linalg

import synthetic
from oracle import brute
from oracle import inputs as oi
from oracle import qsvd_ref as ref
from oracle import quant_ref as qr

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
W0 = synthetic.CONFIGS[0]


@pytest.fixture(scope="module")
def cfg0():
    wq, wk, wv = synthetic.qkv_weights(W0)
    u, s, vt = ref.joint_svd(wq, wk, wv)
    return wq, wk, wv, u, s, vt


# ---------------------------------------------------------------- joint SVD

@pytest.mark.parametrize("beta", [0.0, 0.3, 0.5, 1.0])
@pytest.mark.parametrize("r", [1, 40, 96, 255])
def test_eckart_young_residual(cfg0, r, beta):
    """SVDQuant glossary, 2.3 (Eckart-Young): the rank-r truncation leaves
    squared residual sum_{i>r} sigma_i^2.  Catches a beta split that does
    not multiply back to U_r Sigma_r V_r^T, or mis-sliced q/k/v blocks."""
    wq, wk, wv, u, s, vt = cfg0
    wd, wuq, wuk, wuv = ref.factors(u, s, vt, r, beta)
    res = ref.truncation_residual(wq, wk, wv, wd, wuq, wuk, wuv)
    expect = float(np.sum(s[r:] ** 2))
    assert abs(res - expect) <= 1e-9 * max(expect, 1.0)


def test_singular_vectors_orthonormal(cfg0):
    _, _, _, u, s, vt = cfg0
    r = 96
    assert np.allclose(u[:, :r].T @ u[:, :r], np.eye(r), atol=1e-12)
    assert np.allclose(vt[:r] @ vt[:r].T, np.eye(r), atol=1e-12)
    assert np.all(np.diff(s) <= 0)


def test_spectrum_matches_input_recipe(cfg0):
    """The concatenation's Gram matrix is the sum of the three W W^T, so the
    squared singular values sum to 3E (each W has ||W||_F^2 = E)."""
    _, _, _, u, s, vt = cfg0
    assert abs(np.sum(s ** 2) - 3 * W0.E) < 1e-6 * W0.E


def _full_rank_case(rope_base):
    w = synthetic.replace(W0, r=W0.E)  # rank of an E x 3E matrix is <= E
    wq, wk, wv = synthetic.qkv_weights(w)
    u, s, vt = ref.joint_svd(wq, wk, wv)
    wd, wuq, wuk, wuv = ref.factors(u, s, vt, w.E, 0.5)
    lens = np.array([37, 1, 64])
    xs = [synthetic.sequence_activations(w, b, int(n)) for b, n in enumerate(lens)]
    xq = synthetic.activations(w, len(lens), stream="xnew")
    caches = [ref.latent(x, wd) for x in xs]
    cnew = ref.latent(xq, wd)
    got = ref.decode_materialized(caches, lens, cnew, wuq, wuk, wuv, w.H,
                                  rope_base=rope_base)
    want = ref.attention_uncompressed(xs, lens, xq, wq, wk, wv, w.H,
                                      rope_base=rope_base)
    return got, want


@pytest.mark.parametrize("rope_base", [None, 10000.0])
def test_full_rank_equals_uncompressed(rope_base):
    """At r = E the joint factors are exact, so latent decode must equal
    dense attention on X W_Q, X W_K, X W_V (QSVD digest, Method, Step 1).
    Catches a wrong head split, a transposed up-projection or a wrong
    softmax scale in the latent routine."""
    got, want = _full_rank_case(rope_base)
    assert np.max(np.abs(got - want)) <= 1e-10 * np.max(np.abs(want))


@pytest.mark.parametrize("beta", [0.0, 0.2, 0.8, 1.0])
def test_beta_invariance(cfg0, beta):
    """beta only moves Sigma between the factors (QSVD digest, Method,
    Step 3); without quantisation the output cannot depend on it."""
    wq, wk, wv, u, s, vt = cfg0
    r = 96
    lens = np.array([50, 128])
    xs = [synthetic.sequence_activations(W0, b, int(n)) for b, n in enumerate(lens)]
    xq = synthetic.activations(W0, 2, stream="xnew")

    def run(bt):
        wd, wuq, wuk, wuv = ref.factors(u, s, vt, r, bt)
        return ref.decode_materialized([ref.latent(x, wd) for x in xs], lens,
                                       ref.latent(xq, wd), wuq, wuk, wuv, W0.H)
    a, b = run(0.5), run(beta)
    assert np.max(np.abs(a - b)) <= 1e-11 * np.max(np.abs(a))


# ------------------------------------------------------------------- H2

@pytest.mark.parametrize("n", [1, 2, 8, 64, 256])
def test_hadamard_closed_form(n):
    """Normalised Sylvester Hadamard equals scipy's construction / sqrt(n)
    and is orthogonal."""
    h = ref.hadamard(n)
    assert np.array_equal(h * math.sqrt(n), scipy.linalg.hadamard(n).astype(float))
    assert np.allclose(h @ h.T, np.eye(n), atol=1e-13)


def test_h2_orthogonal_and_kron_layout():
    q3 = synthetic.dct3()
    assert np.allclose(q3 @ q3.T, np.eye(3), atol=1e-14)
    h2 = ref.h2_matrix(4, q3)
    assert np.allclose(h2 @ h2.T, np.eye(12), atol=1e-13)
    # (H (x) Q) vec_row(M) = vec_row(H M Q^T)
    m = np.arange(12, dtype=float).reshape(4, 3) ** 1.5
    lhs = h2 @ m.reshape(-1)
    rhs = (ref.hadamard(4) @ m @ q3.T).reshape(-1)
    assert np.allclose(lhs, rhs, atol=1e-12)


def test_h2_invariance(cfg0):
    """H2 cancels between the factors (QSVD paper notes, 关键设计:
    Y = (X H1^T)(H1 W^d H2^T)(H2 W^u)); without quantisation the output is
    unchanged.  r = 96 = 32 x 3 uses H_32 (x) Q3."""
    wq, wk, wv, u, s, vt = cfg0
    wd, wuq, wuk, wuv = ref.factors(u, s, vt, 96, 0.5)
    h2 = ref.h2_matrix(32, synthetic.dct3())
    rd, rq, rk, rv = ref.rotate_factors(wd, wuq, wuk, wuv, h2)
    lens = np.array([77])
    xs = [synthetic.sequence_activations(W0, 0, 77)]
    xq = synthetic.activations(W0, 1, stream="xnew")
    a = ref.decode_materialized([ref.latent(xs[0], wd)], lens, ref.latent(xq, wd),
                                wuq, wuk, wuv, W0.H)
    b = ref.decode_materialized([ref.latent(xs[0], rd)], lens, ref.latent(xq, rd),
                                rq, rk, rv, W0.H)
    assert np.max(np.abs(a - b)) <= 1e-11 * np.max(np.abs(a))


# ----------------------------------------------------------------- counts

@pytest.mark.parametrize("E,r,L", [(4096, 1536, 8192), (5120, 2304, 100), (256, 96, 1)])
def test_param_and_cache_counts(E, r, L):
    """QSVD paper notes, 关键设计, and QSVD digest, Problem: joint SVD keeps
    4rE weights and rL cache, per-matrix SVD 6rE and 2rL."""
    c = ref.param_counts(E, r, L)
    assert c["joint_params"] == 4 * r * E
    assert c["per_matrix_params"] == 6 * r * E
    assert c["joint_cache"] == r * L
    assert c["per_matrix_cache"] == 2 * r * L


def test_break_even_rank():
    """QSVD digest, Method, Step 1: compression is active below r = 0.75 E."""
    assert ref.compression_active(4096, 3071)
    assert not ref.compression_active(4096, 3072)
    assert ref.compression_active(5120, 3839)
    assert not ref.compression_active(5120, 3840)


def test_cache_ratios_printed():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "cache_ratios.txt"))
            if l.strip() and not l.startswith("#")]
    assert rows
    for E, r, pct in rows:
        got = 100.0 * ref.cache_ratio(int(E), int(r))
        assert abs(got - float(pct)) < 0.005 + 1e-12


# ------------------------------------------------- decode routes, brute force

def test_absorbed_equals_materialized():
    """Absorbing the query (qt_h = W^u_{k,h} q_h) and accumulating values
    in latent space is the same arithmetic reordered."""
    w = synthetic.SHRUNK[1]
    case = oi.build_case(w)
    got = ref.decode_absorbed(case.caches, case.lengths, case.cnew, case.wuq,
                              case.wuk, case.wuv, w.H)
    want = case.reference()
    assert np.max(np.abs(got - want)) <= 1e-11 * np.max(np.abs(want))


@pytest.mark.parametrize("n", [1, 2, 3, 5])
def test_brute_force_loops(n):
    """Scalar loops over the definition on tiny inputs (E=16, H=2, r=6)."""
    g = np.random.default_rng(7 + n)
    E, H, r = 16, 2, 6
    wuq, wuk, wuv = (g.standard_normal((r, E)) for _ in range(3))
    cache = g.standard_normal((n, r))
    qin = g.standard_normal(r)
    want = brute.decode_loops(cache.tolist(), n, qin.tolist(), wuq.tolist(),
                              wuk.tolist(), wuv.tolist(), H)
    got = ref.decode_materialized([cache], [n], qin[None, :], wuq, wuk, wuv, H)[0]
    got2 = ref.decode_absorbed([cache], [n], qin[None, :], wuq, wuk, wuv, H)[0]
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12)
    assert np.allclose(got2, want, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("n", [1, 2, 6])
def test_brute_force_loops_rope(n):
    """Rotary decode against scalar loops: key t at position t, query at
    n - 1, pairs (i, i + d/2).  Pins the position convention independently
    of the dense and latent routines."""
    g = np.random.default_rng(70 + n)
    E, H, r = 16, 2, 6
    wuq, wuk, wuv = (g.standard_normal((r, E)) for _ in range(3))
    cache = g.standard_normal((n, r))
    qin = g.standard_normal(r)
    base = 3.0   # small base: every pair rotates noticeably per step
    want = brute.decode_loops(cache.tolist(), n, qin.tolist(), wuq.tolist(),
                              wuk.tolist(), wuv.tolist(), H, rope_base=base)
    got = ref.decode_materialized([cache], [n], qin[None, :], wuq, wuk, wuv, H,
                                  rope_base=base)[0]
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12)


def test_softmax_special_cases():
    g = np.random.default_rng(3)
    E, H, r = 32, 4, 8
    d_h = E // H
    wuq, wuk, wuv = (g.standard_normal((r, E)) for _ in range(3))
    cache = g.standard_normal((10, r))
    # one token: output is that token's value row
    o1 = ref.decode_materialized([cache], [1], g.standard_normal((1, r)), wuq, wuk, wuv, H)
    assert np.allclose(o1[0], cache[0] @ wuv, atol=1e-12)
    # zero query: uniform weights -> mean of value rows
    o0 = ref.decode_materialized([cache], [10], np.zeros((1, r)), wuq, wuk, wuv, H)
    assert np.allclose(o0[0], (cache @ wuv).mean(axis=0), atol=1e-12)
    # a dominant key gets all the weight
    big = np.zeros((1, E))
    k0 = cache[3] @ wuk
    big[0] = 1e4 * k0
    o2 = ref.decode_materialized([cache], [10], big, wuq, wuk, wuv, H,
                                 qin_is_latent=False)
    v = cache @ wuv
    for h in range(H):
        cols = slice(h * d_h, (h + 1) * d_h)
        scores = (cache @ wuk)[:, cols] @ k0[cols]
        assert np.allclose(o2[0, cols], v[int(np.argmax(scores)), cols], atol=1e-8)


# ------------------------------------------------------------------- RoPE

def test_rope_matches_complex_rotation():
    """Rotate-half pairs (i, i + d/2) are the complex numbers
    a_i + i b_i multiplied by exp(i p theta_i)."""
    g = np.random.default_rng(11)
    d = 128
    v = g.standard_normal((5, d))
    pos = np.array([0, 1, 17, 8191, 32767])
    got = ref.rope(v, pos, 10000.0)
    z = v[:, :d // 2] + 1j * v[:, d // 2:]
    theta = 10000.0 ** (-np.arange(d // 2) * 2.0 / d)
    zr = z * np.exp(1j * pos[:, None] * theta[None, :])
    want = np.concatenate([zr.real, zr.imag], axis=1)
    assert np.allclose(got, want, atol=1e-9)
    assert np.allclose(np.linalg.norm(got, axis=1), np.linalg.norm(v, axis=1))
    assert np.array_equal(ref.rope(v[:1], np.array([0]), 10000.0), v[:1])


def test_rope_relative_position():
    """Scores depend only on the position difference."""
    g = np.random.default_rng(5)
    d = 64
    q = g.standard_normal(d)
    k = g.standard_normal((20, d))
    pos = np.arange(20)
    s0 = ref.rope(k, pos, 10000.0) @ ref.rope(q[None], np.array([19]), 10000.0)[0]
    s1 = ref.rope(k, pos + 1000, 10000.0) @ ref.rope(q[None], np.array([1019]), 10000.0)[0]
    assert np.allclose(s0, s1, atol=1e-9)


# -------------------------------------------------------------- quantiser

def _golden_quant():
    out = []
    for line in open(os.path.join(GOLDEN, "quant_cases.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        head, vals, codes, scales, ovf = [p.strip() for p in line.split("|")]
        bits, group = map(int, head.split())
        out.append((bits, group, np.array(vals.split(), np.float32),
                    np.array(codes.split(), np.int8),
                    np.array(scales.split(), np.float64),
                    np.array(ovf.split(), int).astype(bool)))
    return out


@pytest.mark.parametrize("case", _golden_quant())
def test_quantizer_golden(case):
    bits, group, vals, codes, scales, ovf = case
    got_c, got_s, got_o = qr.quantize(vals, bits, group)
    assert np.array_equal(got_c, codes)
    assert np.array_equal(got_s.astype(np.float64), scales)
    assert np.array_equal(got_o, ovf)


def _f32(x):
    return struct.unpack("f", struct.pack("f", x))[0]


def _f16(x):
    return struct.unpack("e", struct.pack("e", x))[0]


def _scalar_quantizer(vals, bits, group):
    """Independent scalar version: Python floats, struct rounding, round()."""
    qmax = 7 if bits == 4 else 127
    codes, scales = [], []
    for g0 in range(0, len(vals), group):
        grp = [_f32(float(v)) for v in vals[g0:g0 + group]]
        amax = max(abs(v) for v in grp)
        s32 = _f32(amax / qmax)   # fp64 quotient of fp32s rounds correctly
        s16 = _f16(min(s32, 65504.0))
        scales.append(s16)
        for v in grp:
            if s16 == 0.0:
                codes.append(0)
            else:
                codes.append(max(-qmax, min(qmax, round(_f32(v / s16)))))
    return codes, scales


@pytest.mark.parametrize("bits", [4, 8])
def test_quantizer_vs_scalar_version(bits):
    g = np.random.default_rng(bits)
    vals = np.concatenate([
        g.standard_normal(256) * 3,
        np.zeros(32),
        g.standard_normal(32) * 1e-6,
        (np.arange(-64, 64) / 2.0).astype(np.float32),   # exact halves
        g.standard_normal(32) * 5e4,
        np.full(32, 1e-30),                              # subnormal scale
    ]).astype(np.float32)
    group = 32
    codes, scales, _ = qr.quantize(vals, bits, group)
    c2, s2 = _scalar_quantizer(vals.tolist(), bits, group)
    assert codes.tolist() == c2
    assert scales.astype(np.float64).tolist() == s2


def test_quantizer_error_bound_and_packing():
    g = np.random.default_rng(1)
    c = (g.standard_normal((9, 384)) * np.linspace(0.1, 30, 384)).astype(np.float32)
    for bits in (4, 8):
        codes, s16, _ = qr.quantize(c, bits, 128)
        qmax = qr.QMAX[bits]
        assert codes.min() >= -qmax and codes.max() <= qmax
        deq = qr.dequantize(codes, s16, 128)
        sf = np.repeat(s16.astype(np.float32), 128, axis=-1)
        unclamped = np.abs(c / sf) <= qmax
        assert np.all(np.abs(deq - c)[unclamped] <= sf[unclamped] / 2 * (1 + 1e-6))
    codes, _, _ = qr.quantize(c, 4, 128)
    assert np.array_equal(qr.unpack_int4(qr.pack_int4(codes)), codes)
    p = qr.pack_int4(np.array([[1, -1, -8, 7]], np.int8))
    assert p.tolist() == [[0xF1, 0x78]]


# ---------------------------------------------------------- output projection

def _wo(E, seed):
    return np.random.default_rng(seed).standard_normal((E, E)) / math.sqrt(E)


@pytest.mark.parametrize("cfg", [1, 2, 3])
def test_fold_equals_projected_materialized(cfg):
    """sum_h z_h (W^u_{v,h} W_{O,h}) is the attention of the materialised
    route (values rebuilt, heads concatenated) times W_O, with and without
    rotary embedding; an empty sequence gives a zero row."""
    w = synthetic.SHRUNK[cfg]
    case = oi.build_case(w)
    lengths = case.lengths.copy()
    lengths[-1] = 0
    wo = _wo(w.E, 4)
    rb = w.rope_base if w.rope else None
    want = ref.output_projection(
        ref.decode_materialized(case.caches, lengths, case.cnew, case.wuq, case.wuk, case.wuv, w.H,
                                rope_base=rb), wo)
    z = ref.decode_absorbed_latents(case.caches, lengths, case.cnew, case.wuq, case.wuk, w.H,
                                    rope_base=rb)
    got = ref.decode_folded(z, ref.fold_value_output(case.wuv, wo, w.H))
    assert np.max(np.abs(got - want)) <= 1e-11 * np.max(np.abs(want))
    assert np.all(got[-1] == 0.0)


def test_fold_with_identity_output_projection():
    """W_O = I: F_h is W^u_{v,h} placed in head h's columns, zero elsewhere
    (fixes which rows of W_O and which columns of W^u_v meet)."""
    E, H, r = 96, 3, 40
    wuv = np.random.default_rng(2).standard_normal((r, E))
    f = ref.fold_value_output(wuv, np.eye(E), H)
    d_h = E // H
    for h in range(H):
        blk = f[h * r:(h + 1) * r]
        assert np.array_equal(blk[:, h * d_h:(h + 1) * d_h], wuv[:, h * d_h:(h + 1) * d_h])
        mask = np.ones(E, bool)
        mask[h * d_h:(h + 1) * d_h] = False
        assert np.all(blk[:, mask] == 0.0)


def test_output_projection_permutation():
    """A permutation W_O moves columns: y[:, perm[j]] = o[:, j]."""
    g = np.random.default_rng(8)
    o = g.standard_normal((3, 12))
    perm = g.permutation(12)
    wo = np.zeros((12, 12))
    wo[np.arange(12), perm] = 1.0
    y = ref.output_projection(o, wo)
    assert np.array_equal(y[:, perm], o)


# ------------------------------------------------------------- prefill attention

@pytest.mark.parametrize("cfg", [1, 2])
def test_prefill_last_rows_are_decode_steps(cfg):
    """Row t of the causal prefill is the decode step of a sequence of t + 1
    tokens whose current latent is row t (rotary: query at position t)."""
    w = synthetic.SHRUNK[cfg]
    case = oi.build_case(w)
    c = case.caches[0]
    n = c.shape[0]
    rb = w.rope_base if w.rope else None
    pre = ref.prefill_attention(c, case.wuq, case.wuk, case.wuv, w.H, rope_base=rb)
    for t in (0, 1, n // 2, n - 1):
        dec = ref.decode_materialized([c[:t + 1]], [t + 1], c[t:t + 1], case.wuq, case.wuk, case.wuv,
                                      w.H, rope_base=rb)
        assert np.max(np.abs(pre[t] - dec[0])) <= 1e-11 * np.max(np.abs(dec))


def test_prefill_brute_force_loops():
    """Scalar loops over tokens, heads and channels on a tiny case."""
    g = np.random.default_rng(6)
    L, r, H, d_h = 5, 6, 2, 4
    E = H * d_h
    c = g.standard_normal((L, r))
    wuq, wuk, wuv = (g.standard_normal((r, E)) for _ in range(3))
    got = ref.prefill_attention(c, wuq, wuk, wuv, H)
    tau = 1.0 / math.sqrt(d_h)
    for t in range(L):
        for h in range(H):
            qv = [sum(c[t][j] * wuq[j][h * d_h + i] for j in range(r)) for i in range(d_h)]
            logits = []
            for u in range(t + 1):
                kv = [sum(c[u][j] * wuk[j][h * d_h + i] for j in range(r)) for i in range(d_h)]
                logits.append(tau * sum(qv[i] * kv[i] for i in range(d_h)))
            mx = max(logits)
            ws = [math.exp(x - mx) for x in logits]
            for i in range(d_h):
                num = sum(ws[u] * sum(c[u][j] * wuv[j][h * d_h + i] for j in range(r)) for u in range(t + 1))
                assert abs(got[t][h * d_h + i] - num / sum(ws)) <= 1e-12 * (1 + abs(num / sum(ws)))
