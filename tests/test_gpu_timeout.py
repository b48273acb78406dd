"""The bounded-wait failure path of the tensor-core split kernel, made to run
without any fault.

Every wait inside a kernel gives up after 2 s, records QSVD_STATUS_TIMEOUT in
the workspace status word, and the kernel then waits (again bounded) for its
own copies and MMAs in flight, frees its tensor memory and returns.  Through
the testing hook the softmax warps first wait on a barrier that nothing
releases (limit 1 ms), so the wait expires on every CTA of a tiny decode: the
call must come back with the status bit set, and the next decode without the
injection must be exact again (the context stays usable)."""
import time

import numpy as np
import pytest
import torch

import rank_joint_qkv_b200 as q
import synthetic
from oracle import inputs as oi
from tests.gpu_util import GpuCase, rel_err

pytestmark = pytest.mark.gpu


def test_expired_score_wait_sets_timeout_and_returns(cuda_ok):
    case = oi.build_case(synthetic.SHRUNK[1])
    g = GpuCase(case, kernel=q.QSVD_KERNEL_TCGEN05_CTA)
    try:
        q.qsvd_testing_set_score_wait_ns(1_000_000)
        t0 = time.perf_counter()
        _, ws = g.decode()          # synchronises
        dt = time.perf_counter() - t0
        assert q.status_word(ws) & q.QSVD_STATUS_TIMEOUT
        assert dt < 30.0            # every other wait gave up within its own 2 s limit
    finally:
        q.qsvd_testing_set_score_wait_ns(0)
    got, ws = g.decode()
    assert q.status_word(ws) == 0
    assert rel_err(got, case.reference()) <= 2e-3
