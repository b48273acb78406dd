"""Pins of the oracle's beta search (``oracle.beta_ref``), no GPU.

* One-token sequences: the softmax weight is 1, so the decode output is the
  latent times W^u_v and the objective has the closed form
  sum_d ||(c_d - Q(c_d)) W^u_v||^2.
* The golden-section search finds the minimiser of a quadratic to its
  bracket's width, stays on a boundary minimum, and evaluates one new point
  per refinement step.
* On the seeded outlier workload the objective is positive, depends on
  beta, is smaller for int8 than for int4 at every beta, and the search's
  beta is no worse than the pages' default split of 0.5.
"""
import math

import numpy as np
import pytest

import synthetic
from oracle import beta_ref as br
from oracle import inputs as oi
from oracle import quant_ref as qr
from oracle import qsvd_ref as ref


def _setup(seq_len, B=3):
    w = synthetic.replace(synthetic.SHRUNK[1], B=B, L=seq_len)
    wq, wk, wv = synthetic.qkv_weights(w)
    u, s, vt = ref.joint_svd(wq, wk, wv)
    xs = [oi.from_device_dtype(oi.to_device_dtype(synthetic.sequence_activations(w, b, seq_len), "f16"),
                               "f16") for b in range(B)]
    return w, (u, s, vt), xs, np.full(B, seq_len, np.int32)


def test_one_token_closed_form():
    w, (u, s, vt), xs, lens = _setup(1)
    for beta in (0.0, 0.35, 1.0):
        got = br.calibration_objective(u, s, vt, w.r, beta, xs, lens, w.H, bits=4, group=128)
        wd, _, _, wuv = br.beta_weights(u, s, vt, w.r, beta, "f16")
        want = 0.0
        for x in xs:
            c = (x @ wd).astype(np.float32)
            codes, sc, _ = qr.quantize(c, 4, 128)
            dq = qr.dequantize(codes, sc, 128).astype(np.float64)
            want += float(np.sum(((c.astype(np.float64) - dq) @ wuv) ** 2))
        assert want > 0
        assert abs(got - want) <= 1e-9 * want


def test_golden_section_quadratic():
    calls = []

    def f(b):
        calls.append(b)
        return (b - 0.37) ** 2

    grid = [i / 10 for i in range(11)]
    beta, val, evals = br.search(f, grid, refine=40)
    assert abs(beta - 0.37) < 1e-7
    assert val == pytest.approx((beta - 0.37) ** 2)
    assert len(calls) == len(set(calls)) == len(evals)
    assert len(evals) == len(grid) + 40 + 1       # one new point per step after the first


def test_search_keeps_boundary_minimum():
    beta, val, _ = br.search(lambda b: b + 1.0, [0.0, 0.5, 1.0], refine=10)
    assert beta == 0.0 and val == 1.0


@pytest.fixture(scope="module")
def outlier_case():
    return _setup(160)


def test_objective_depends_on_beta(outlier_case):
    w, (u, s, vt), xs, lens = outlier_case
    grid = [0.0, 0.25, 0.5, 0.75, 1.0]
    j4 = [br.calibration_objective(u, s, vt, w.r, b, xs, lens, w.H, bits=4, group=128) for b in grid]
    j8 = [br.calibration_objective(u, s, vt, w.r, b, xs, lens, w.H, bits=8, group=128) for b in grid]
    assert all(v > 0 for v in j4 + j8)
    assert all(a < b for a, b in zip(j8, j4))
    assert max(j4) > 1.5 * min(j4)               # beta moves the quantisation error


def test_search_no_worse_than_even_split(outlier_case):
    w, (u, s, vt), xs, lens = outlier_case

    def obj(b):
        return br.calibration_objective(u, s, vt, w.r, b, xs, lens, w.H, bits=4, group=128)

    beta, val, evals = br.search(obj, [0.0, 0.25, 0.5, 0.75, 1.0], refine=4)
    assert val <= evals[0.5]
    assert 0.0 <= beta <= 1.0 and math.isfinite(val)
