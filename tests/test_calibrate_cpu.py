"""Host logic of the beta search (``rank_joint_qkv_b200.calibrate.search_beta``),
no GPU: on objectives given as plain functions it must evaluate the same
points in the same order and pick the same beta as the oracle's search
(``oracle.beta_ref.search``), written separately from the same description
(grid, then golden-section between the best grid point's neighbours)."""
import numpy as np
import pytest

from oracle import beta_ref as br
from rank_joint_qkv_b200.calibrate import search_beta


def _recorded(fn):
    calls = []

    def f(b):
        calls.append(b)
        return fn(b)
    return f, calls


def _noisy(seed):
    g = np.random.default_rng(seed)
    knots = g.uniform(0.5, 2.0, size=41)
    return lambda b: float(np.interp(b, np.linspace(0, 1, 41), knots)) + (b - 0.6) ** 2


@pytest.mark.parametrize("fn", [lambda b: (b - 0.37) ** 2, lambda b: abs(b - 0.9), lambda b: -b,
                                _noisy(1), _noisy(2), _noisy(3)])
@pytest.mark.parametrize("grid,refine", [([i / 10 for i in range(11)], 8), ([0.0, 0.25, 0.5, 0.75, 1.0], 12),
                                         ([0.0, 1.0], 5)])
def test_same_evaluations_as_oracle(fn, grid, refine):
    f1, c1 = _recorded(fn)
    f2, c2 = _recorded(fn)
    b1, v1, e1 = search_beta(f1, grid, refine)
    b2, v2, e2 = br.search(f2, grid, refine)
    assert c1 == c2
    assert (b1, v1) == (b2, v2) and e1 == e2


def test_quadratic_minimum_found():
    beta, val, _ = search_beta(lambda b: (b - 0.37) ** 2, refine=40)
    assert abs(beta - 0.37) < 1e-7
