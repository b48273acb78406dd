"""Prefill parity: the latent rows of many tokens at once (one tensor-core
GEMM x W^d with rounding or quantisation fused), scattered to their cache
rows.

As in the append tests, the stored bytes are checked bit-exactly against the
oracle's quantiser wherever the float32 latent is exact (W^d = I, or integer
activations times dyadic weights); a general projection is compared with the
fp64 oracle with a tolerance, and its stored rows must be exactly the
rounding / quantisation of the latent the kernel reports.
"""
import numpy as np
import pytest
import torch

import rank_joint_qkv_b200 as q
from oracle import inputs as oi
from oracle import quant_ref as qr
from tests.test_gpu_append import adversarial_x, expected_rows, run_append

pytestmark = pytest.mark.gpu
DEV = "cuda"
ROWB = {"f32": 4, "f16": 2, "bf16": 2, "i8": 1}


def run_prefill(E, r, B, max_len, x, wd, cache_dtype, weight, dst, *, sentinel=0x5A):
    dims = q.make_dims(E, E // 128, 128, r, B, max_len, cache=cache_dtype, weight=weight)
    wdt = oi.as_torch(oi.to_device_dtype(wd, weight), weight).to(DEV)
    wu = torch.zeros((r, E), dtype=wdt.dtype, device=DEV)
    packed = q.qsvd_prepare_weights(dims, wdt, wu, wu, wu)
    xt = oi.as_torch(oi.to_device_dtype(x, weight), weight).to(DEV)
    rowb = r // 2 if cache_dtype == "i4" else ROWB[cache_dtype] * r
    cache = torch.full((B, max_len, rowb), sentinel, dtype=torch.uint8, device=DEV)
    scales = (torch.zeros((B, max_len, r // 128), dtype=torch.float16, device=DEV)
              if cache_dtype in ("i8", "i4") else None)
    c_out = torch.zeros((x.shape[0], r), dtype=torch.float32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    dst_t = torch.from_numpy(np.asarray(dst, np.int32)).to(DEV)
    q.qsvd_prefill_latent(dims, packed, xt, dst_t, cache, scales, c_out, status)
    torch.cuda.synchronize()
    return (cache.cpu().numpy().reshape(B * max_len, rowb),
            None if scales is None else scales.cpu().numpy().reshape(B * max_len, -1),
            c_out.cpu().numpy(), int(status.item()))


def scatter(n, B, max_len, g):
    """Distinct destination rows for n tokens, in shuffled order."""
    return g.permutation(B * max_len)[:n].astype(np.int32)


@pytest.mark.parametrize("cache_dtype", ["i4", "i8", "f16", "bf16", "f32"])
@pytest.mark.parametrize("weight", ["f16", "bf16"])
def test_identity_projection_bit_exact(cuda_ok, cache_dtype, weight):
    """W^d = I (E = r = 512): the latent is x, every stored byte is fixed;
    300 rows (a ragged last tile), two column blocks, scattered rows."""
    E = r = 512
    B, max_len, n = 3, 128, 300
    g = np.random.default_rng(11)
    x = np.concatenate([adversarial_x(3, E, g), (g.standard_normal((n - 3, E)) * 2)])
    x = oi.from_device_dtype(oi.to_device_dtype(x, weight), weight).astype(np.float32)
    dst = scatter(n, B, max_len, g)
    cache, scales, c_out, st = run_prefill(E, r, B, max_len, x, np.eye(E), cache_dtype, weight, dst)
    assert np.array_equal(c_out, x)
    rows, s16 = expected_rows(x, cache_dtype, 128)
    assert np.array_equal(cache[dst], rows)
    if s16 is not None:
        assert np.array_equal(scales[dst].view(np.uint16), s16.view(np.uint16))
    untouched = np.setdiff1d(np.arange(B * max_len), dst)
    assert np.all(cache[untouched] == 0x5A)
    assert st == 0


@pytest.mark.parametrize("cache_dtype,r", [("i4", 768), ("i8", 768), ("f16", 1536)])
def test_dyadic_projection_bit_exact_llava_shapes(cuda_ok, cache_dtype, r):
    """E = 4096 with integer activations and weights on a 1/8 grid: x W^d is
    exact in float32 in any summation order."""
    E, B, max_len, n = 4096, 2, 160, 200
    g = np.random.default_rng(5)
    x = g.integers(-3, 4, size=(n, E)).astype(np.float32)
    wd = g.integers(-16, 17, size=(E, r)).astype(np.float64) / 8.0
    exact = x.astype(np.float64) @ wd
    assert np.max(np.abs(exact)) < 2 ** 20
    dst = scatter(n, B, max_len, g)
    cache, scales, c_out, st = run_prefill(E, r, B, max_len, x, wd, cache_dtype, "f16", dst)
    assert np.array_equal(c_out.astype(np.float64), exact)
    rows, s16 = expected_rows(exact.astype(np.float32), cache_dtype, 128)
    assert np.array_equal(cache[dst], rows)
    if s16 is not None:
        assert np.array_equal(scales[dst].view(np.uint16), s16.view(np.uint16))
    assert st == 0


@pytest.mark.parametrize("cache_dtype", ["f16", "i4"])
@pytest.mark.parametrize("weight", ["f16", "bf16"])
def test_general_projection(cuda_ok, cache_dtype, weight):
    """Random x and W^d: the latent matches the fp64 product of the rounded
    operands to float32 accumulation error, and the stored rows are exactly
    the rounding / quantisation of the latent the kernel reports."""
    E, r, B, max_len, n = 1024, 512, 2, 256, 383
    g = np.random.default_rng(3)
    x = oi.from_device_dtype(oi.to_device_dtype(g.standard_normal((n, E)), weight), weight)
    wd = oi.from_device_dtype(oi.to_device_dtype(g.standard_normal((E, r)) / np.sqrt(E), weight), weight)
    dst = scatter(n, B, max_len, g)
    cache, scales, c_out, st = run_prefill(E, r, B, max_len, x, wd, cache_dtype, weight, dst)
    want = x.astype(np.float64) @ wd.astype(np.float64)
    err = np.max(np.abs(c_out - want)) / np.sqrt(np.mean(want ** 2))
    assert err <= 1e-5, err
    rows, s16 = expected_rows(c_out, cache_dtype, 128)
    assert np.array_equal(cache[dst], rows)
    if s16 is not None:
        assert np.array_equal(scales[dst].view(np.uint16), s16.view(np.uint16))
    assert st == 0


def test_matches_append_path(cuda_ok):
    """The same tokens through qsvd_append_latent: the same latent to float32
    accumulation error (the GEMV and the GEMM sum in different orders)."""
    E, r, B = 1024, 512, 3
    g = np.random.default_rng(9)
    x = oi.from_device_dtype(oi.to_device_dtype(g.standard_normal((B, E)), "f16"), "f16")
    wd = g.standard_normal((E, r)) / np.sqrt(E)
    _, _, c_app, _ = run_append(E, r, B, x, wd, "f16", "f16")
    _, _, c_pre, _ = run_prefill(E, r, B, 8, x, wd, "f16", "f16", np.arange(B) * 8)
    assert np.max(np.abs(c_pre - c_app)) <= 1e-5 * np.sqrt(np.mean(c_app.astype(np.float64) ** 2))


def test_rows_out_of_range_skipped_and_flagged(cuda_ok):
    E = r = 256
    B, max_len, n = 2, 4, 5
    g = np.random.default_rng(1)
    x = oi.from_device_dtype(oi.to_device_dtype(g.standard_normal((n, E)), "f16"), "f16")
    dst = np.array([0, -1, 7, 8, 3], np.int32)          # -1 and 8 are outside [0, B * max_len)
    cache, _, c_out, st = run_prefill(E, r, B, max_len, x, np.eye(E), "f16", "f16", dst)
    assert st & q.QSVD_STATUS_POS_OOB
    rows, _ = expected_rows(x.astype(np.float32), "f16", 128)
    for i in (0, 2, 4):
        assert np.array_equal(cache[dst[i]], rows[i])
    for row in (1, 2, 4, 5, 6):
        assert np.all(cache[row] == 0x5A)


def test_zero_rows_is_a_no_op(cuda_ok):
    E = r = 256
    cache, _, _, st = run_prefill(E, r, 1, 4, np.zeros((0, E), np.float32), np.eye(E), "f16", "f16",
                                  np.zeros(0, np.int32))
    assert np.all(cache == 0x5A) and st == 0
