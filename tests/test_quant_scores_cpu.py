"""Host-side replay of the quantised path's score arithmetic (prologue.cu
k_quant_query, split_tc.cu S MMAs and softmax), no GPU.

The absorbed query of one (sequence, head) enters the integer tensor cores
as three int8 parts under one power-of-two scale sq:
q ~ sq (p0 + p1 / 128 + p2 / 16384).  Per 128-channel group the MMAs add
S_k = sum_c code_c p_k,c onto a TMEM word preset to the bits 0x4B400000
(1.5 x 2^23), so the word read back as a float is 1.5 x 2^23 + S_k exactly;
the softmax subtracts the three biases and weights the parts in fp32.
These tests restate those formulas in float32 and check the claims the
kernels rest on: every part fits int8, the residual is within sq 2^-15,
|S_k| stays below 2^22 for any codes (so the biased word keeps its
exponent and the int32 sum cannot carry into it), and the combine returns
S0 + S1 / 128 + S2 / 16384 to fp32 rounding.
"""
import numpy as np
import pytest

F32 = np.float32
BIAS_BITS = 0x4B400000


def quant_query(row):
    """k_quant_query's formulas, float32 throughout."""
    row = np.asarray(row, dtype=F32)
    m = F32(np.max(np.abs(row))) if row.size else F32(0)
    f = F32(m / F32(127))
    if f > 0:
        bits = (np.array(f, dtype=F32).view(np.uint32) + np.uint32(0x007FFFFF)) & np.uint32(0xFF800000)
        sq = F32(np.array(bits, dtype=np.uint32).view(F32))
    else:
        sq = F32(1)
    isq = F32(F32(1) / sq)
    q0 = np.rint(row * isq).astype(F32)
    r1 = (row - sq * q0).astype(F32)
    q1 = np.rint(r1 * isq * F32(128)).astype(F32)
    r2 = (r1 - sq * F32(1 / 128) * q1).astype(F32)
    q2 = np.rint(r2 * isq * F32(16384)).astype(F32)
    return sq, q0, q1, q2, r1, r2


def biased(s):
    """The TMEM word after the integer MMAs, read as a float."""
    w = (np.int64(BIAS_BITS) + np.asarray(s, dtype=np.int64))
    assert np.all((w >= 0) & (w < 2 ** 31)), "the int32 sum overflows"
    return w.astype(np.uint32).view(F32)


def combine(a0, a1, a2):
    """g0 = a0 - 1.5 2^23 (1 + 2^-7 + 2^-14); two fmas (each one rounding:
    the float64 sum of these operands is exact)."""
    g0 = (a0 - F32(12681984.0)).astype(F32)
    t = (a1.astype(np.float64) / 128 + g0.astype(np.float64)).astype(F32)
    return (a2.astype(np.float64) / 16384 + t.astype(np.float64)).astype(F32)


ROWS = {
    "gaussian": lambda g: g.standard_normal(768).astype(F32),
    "outlier": lambda g: np.where(np.arange(768) % 97 == 0, 40.0, 1.0).astype(F32) * g.standard_normal(768).astype(F32),
    "max-is-127-times-a-power-of-two": lambda g: np.concatenate([[F32(127 * 2.0 ** -3)], g.uniform(-1, 1, 767)]).astype(F32),
    "tiny (subnormal max / 127)": lambda g: (g.uniform(-1, 1, 256) * 1e-37).astype(F32),
    "huge": lambda g: (g.uniform(-1, 1, 256) * 3e38).astype(F32),
    "zeros": lambda g: np.zeros(256, dtype=F32),
}


@pytest.mark.parametrize("name", list(ROWS))
def test_query_parts_fit_int8_and_the_residual_is_within_sq_2_pow_minus_15(name):
    row = ROWS[name](np.random.default_rng(7))
    sq, q0, q1, q2, r1, r2 = quant_query(row)
    m = float(np.max(np.abs(row)))
    # sq is a power of two, at least m / 127 (1 for an all-zero row)
    mant, _ = np.frexp(np.float64(sq))
    assert mant == 0.5
    assert float(sq) * 127 >= m * (1 - 2 ** -23)
    if m / 127 >= 2.0 ** -126:
        assert float(sq) < 2 * m / 127 * (1 + 2 ** -22)
    elif m > 0:
        # m / 127 subnormal (the library keeps denormals): sq is the smallest
        # normal, 2^-126, and the residual below is absolute, 2^-141
        assert sq == F32(2.0 ** -126)
    assert np.all(np.abs(q0) <= 127) and np.all(np.abs(q1) <= 64) and np.all(np.abs(q2) <= 64)
    # the two subtractions are exact (Sterbenz): float64 gives the same bits
    s64 = np.float64(sq)
    assert np.array_equal(r1.astype(np.float64), row.astype(np.float64) - s64 * q0)
    assert np.array_equal(r2.astype(np.float64), r1.astype(np.float64) - s64 / 128 * q1)
    approx = s64 * (q0.astype(np.float64) + q1 / 128.0 + q2 / 16384.0)
    err = np.max(np.abs(row.astype(np.float64) - approx))
    assert err <= s64 * 2.0 ** -15
    if name == "zeros":
        assert sq == 1 and not q0.any() and not q1.any() and not q2.any()


@pytest.mark.parametrize("qmax", [7, 127])
def test_group_sums_keep_the_biased_word_in_one_exponent(qmax):
    """Worst case per group: 128 codes at +-qmax against parts at their
    limits.  1.5 2^23 + S must lie in [2^23, 2^24), where floats are the
    integers, and the int32 sum must not carry into the exponent bits."""
    worst = 128 * qmax * 127
    assert worst < 2 ** 22
    s = np.array([-worst, -1, 0, 1, worst, -(2 ** 22) + 1, 2 ** 22 - 1], dtype=np.int64)
    a = biased(s)
    assert np.array_equal(a.astype(np.float64), 1.5 * 2 ** 23 + s)
    assert np.all((a >= 2 ** 23) & (a < 2 ** 24))


@pytest.mark.parametrize("qmax", [7, 127])
def test_combine_returns_the_weighted_part_sums(qmax):
    g = np.random.default_rng(11)
    row = g.standard_normal(128).astype(F32) * 3
    sq, q0, q1, q2, _, _ = quant_query(row)
    parts = np.stack([q0, q1, q2]).astype(np.int64)            # [3][128 channels]
    codes = g.integers(-qmax, qmax + 1, size=(4096, 128))      # tokens x channels
    codes[0] = qmax * np.sign(parts[0] + 0.5)                  # a token at the sum's limit
    s = codes @ parts.T                                        # exact int64 [tokens][3]
    assert np.max(np.abs(s)) < 2 ** 22
    got = combine(biased(s[:, 0]), biased(s[:, 1]), biased(s[:, 2])).astype(np.float64)
    want = s[:, 0] + s[:, 1] / 128.0 + s[:, 2] / 16384.0
    # two fp32 roundings of numbers below 2^22
    assert np.max(np.abs(got - want)) <= 2 * 2.0 ** -24 * (2 ** 22)
    # against the float dot product with the query itself (in units of sq):
    # off by at most sum |code| x the residual bound 2^-15
    exact = codes @ (row.astype(np.float64) / float(sq))
    assert np.max(np.abs(exact - want)) <= 128 * qmax * 2.0 ** -15


def test_the_combine_constant_is_the_three_biases():
    assert 12681984.0 == 1.5 * 2 ** 23 * (1 + 2 ** -7 + 2 ** -14)
    assert np.array(1.5 * 2 ** 23, dtype=F32).view(np.uint32) == BIAS_BITS


def test_the_replay_uses_the_kernels_constants():
    """The constants above are the ones in the sources: a change there has
    to be carried into this replay."""
    import os
    import re
    csrc = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "rank_joint_qkv_b200", "csrc")
    pro = open(os.path.join(csrc, "prologue.cu")).read()
    sp = open(os.path.join(csrc, "split_tc.cu")).read()
    assert "const float f = m / 127.f;" in pro
    assert "(__float_as_uint(f) + 0x007FFFFFu) & 0xFF800000u" in pro
    for frag in ("rintf(v * isq)", "rintf(r1 * isq * 128.f)", "r1 - sq * (1.f / 128.f) * q1",
                 "rintf(r2 * isq * 16384.f)"):
        assert frag in pro, frag
    assert re.search(r"kBias\s*=\s*0x4B400000u", sp)
    assert "a0[e] - 12681984.f" in sp
    assert "fmaf(a2[e], 1.f / 16384.f, fmaf(a1[e], 1.f / 128.f, g0))" in sp
