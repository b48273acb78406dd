"""Parity of the split-exponent (beta) search run through the library
(``rank_joint_qkv_b200.calibrate``) with the oracle's (``oracle.beta_ref``).

The objective sum_d ||Y_d - Y'_d||^2 is compared at fixed betas, not the
search's choice: the objective is a sum over discrete quantisation decisions
and is not smooth in beta, so two correct evaluations a hair apart can send a
search down different brackets.  Both sides get the same float32 singular
vectors and the same 16-bit activations.

Bars: relative difference of the objective <= 2e-3 with the CUDA-core split
kernel (float32 throughout; what remains is the rare quantisation code that
the two latent sums put on different sides of a rounding boundary), 5e-2
with the tensor-core kernel for the quantised cache (its P and query parts
are 16-bit: ~1e-3 of the output, against a quantisation error of a few
percent).  The search is checked for its own contract: the best evaluation,
no worse than the even split, one new evaluation per refinement step.
"""
import numpy as np
import pytest
import torch

import rank_joint_qkv_b200 as q
import synthetic
from oracle import beta_ref as br
from oracle import inputs as oi
from oracle import qsvd_ref as ref
from rank_joint_qkv_b200.calibrate import BetaObjective, search_beta

pytestmark = pytest.mark.gpu
GRID = [0.0, 0.25, 0.5, 0.75, 1.0]


def _setup(h2_m=0, r=256, B=3, L=160, cache="i4"):
    w = synthetic.replace(synthetic.SHRUNK[1], B=B, L=L, r=r)
    wq, wk, wv = synthetic.qkv_weights(w)
    u, s, vt = ref.joint_svd(wq, wk, wv)
    u32 = u[:, :r].astype(np.float32)
    vt32 = vt[:r].astype(np.float32)
    lens = synthetic.lengths(w)
    lens[-1] = L // 2 + 3                            # a ragged sequence
    xs = [oi.from_device_dtype(oi.to_device_dtype(synthetic.sequence_activations(w, b, int(n)), "f16"),
                               "f16") for b, n in enumerate(lens)]
    h2 = None if not h2_m else ref.h2_matrix(r // h2_m, np.eye(h2_m))

    def oracle(beta):
        return br.calibration_objective(u32.astype(np.float64), s, vt32.astype(np.float64), r, beta, xs,
                                        lens, w.H, bits=4 if cache == "i4" else 8, group=128, h2=h2)

    x_dev = torch.from_numpy(np.concatenate(xs).astype(np.float16)).cuda()

    def gpu(kernel):
        return BetaObjective(torch.from_numpy(u32), s[:r], torch.from_numpy(vt32), x_dev, lens, w.H,
                             cache=cache, h2_q=None if not h2_m else np.eye(h2_m), h2_m=h2_m,
                             kernel=kernel)

    return oracle, gpu


@pytest.mark.parametrize("h2_m,cache", [(0, "i4"), (2, "i4"), (0, "i8")])
def test_objective_matches_oracle_cuda_cores(cuda_ok, h2_m, cache):
    oracle, gpu = _setup(h2_m=h2_m, cache=cache)
    obj = gpu(q.QSVD_KERNEL_SIMT)
    for beta in GRID:
        want, got = oracle(beta), obj(beta)
        assert want > 0
        assert abs(got - want) <= 2e-3 * want, (beta, got, want)
    assert obj.status_word() == 0


def test_objective_matches_oracle_tensor_cores(cuda_ok):
    oracle, gpu = _setup()
    obj = gpu(q.QSVD_KERNEL_AUTO)
    for beta in GRID:
        want, got = oracle(beta), obj(beta)
        assert abs(got - want) <= 5e-2 * want, (beta, got, want)


def test_search_contract(cuda_ok):
    _, gpu = _setup()
    obj = gpu(q.QSVD_KERNEL_SIMT)
    beta, val, evals = search_beta(obj, GRID, refine=4)
    assert val == min(evals.values()) and evals[beta] == val
    assert val <= evals[0.5]
    assert len(evals) == obj.evaluations == len(GRID) + 4 + 1
