"""Append parity: latent projection, optional online H2, quantise/pack.

The quantise/pack step is bit-exact.  To give both sides the identical
float32 latent, the projection is made exact: either W^d = s*I (s a power of
two) or small-integer activations times dyadic weights, whose fp32 sums are
exact in any order.  The rotation H2 and general projections are floating
point and are compared with a tolerance.
"""
import numpy as np
import pytest
import torch

import rank_joint_qkv_b200 as q
import synthetic
from oracle import inputs as oi
from oracle import qsvd_ref as ref
from oracle import quant_ref as qr

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run_append(E, r, B, x, wd, cache_dtype, weight, *, group=128, h2=False, h2_q=None,
               h2_m=0, max_len=8, pos=None, wu=None):
    dims = q.make_dims(E, E // 128 if E % 128 == 0 else 1, 128 if E % 128 == 0 else E, r, B,
                       max_len, cache=cache_dtype, weight=weight, group=group, h2=h2, h2_m=h2_m)
    wdt = oi.as_torch(oi.to_device_dtype(wd, weight), weight).to(DEV)
    if wu is None:
        wu = np.zeros((r, E))
    wut = oi.as_torch(oi.to_device_dtype(wu, weight), weight).to(DEV)
    packed = q.qsvd_prepare_weights(dims, wdt, wut, wut, wut, h2_q=h2_q)
    xt = oi.as_torch(oi.to_device_dtype(x, weight), weight).to(DEV)
    if pos is None:
        pos = np.arange(B) % max_len
    post = torch.from_numpy(np.asarray(pos, np.int32)).to(DEV)
    rowb = {"f32": 4 * r, "f16": 2 * r, "bf16": 2 * r, "i8": r, "i4": r // 2}[cache_dtype]
    cache = torch.zeros((B, max_len, rowb), dtype=torch.uint8, device=DEV)
    scales = torch.zeros((B, max_len, r // group), dtype=torch.float16, device=DEV) \
        if cache_dtype in ("i8", "i4") else None
    c_out = torch.zeros((B, r), dtype=torch.float32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    q.qsvd_append_latent(dims, packed, xt, post, cache, scales, c_out, status)
    torch.cuda.synchronize()
    return (cache.cpu().numpy(), None if scales is None else scales.cpu().numpy(),
            c_out.cpu().numpy(), int(status.item()))


def expected_rows(c32, cache_dtype, group):
    if cache_dtype in ("i8", "i4"):
        codes, s16, _ = qr.quantize(c32, 4 if cache_dtype == "i4" else 8, group)
        rows = qr.pack_int4(codes) if cache_dtype == "i4" else codes.view(np.uint8)
        return rows.view(np.uint8), s16
    dev = oi.to_device_dtype(c32.astype(np.float64), cache_dtype)
    return np.ascontiguousarray(dev).view(np.uint8).reshape(c32.shape[0], -1), None


def adversarial_x(B, E, g):
    x = (g.standard_normal((B, E)) * 3).astype(np.float32)
    x[0, :128] = 0.0                                  # an all-zero group
    x[0, 128:256] = (np.arange(128) - 64) / 2.0        # exact halves -> ties
    x[1, :128] = g.standard_normal(128) * 1e-5         # fp16-subnormal scales
    x[1, 128:256] = np.clip(g.standard_normal(128), -3, 3) * 1e4   # large values
    if B > 2:
        x[2, :] = np.float16(1.0)                      # constant row
    return np.asarray(x.astype(np.float16), np.float32)   # values exact in fp16


@pytest.mark.parametrize("cache_dtype", ["i4", "i8", "f16", "bf16", "f32"])
@pytest.mark.parametrize("weight", ["f16", "f32"])
def test_identity_projection_bit_exact(cuda_ok, cache_dtype, weight):
    """W^d = I: the latent is x itself, so every stored byte is fixed."""
    B, E = 4, 512
    g = np.random.default_rng(42)
    x = adversarial_x(B, E, g)
    cache, scales, c_out, st = run_append(E, E, B, x, np.eye(E), cache_dtype, weight)
    assert np.array_equal(c_out, x)
    rows, s16 = expected_rows(x, cache_dtype, 128)
    for b in range(B):
        assert np.array_equal(cache[b, b], rows[b]), f"row {b}"
        if s16 is not None:
            assert np.array_equal(scales[b, b].view(np.uint16), s16[b].view(np.uint16))
    assert st == 0


def test_scale_saturation_flag(cuda_ok):
    B, E = 2, 256
    x = np.zeros((B, E), np.float32)
    x[0, :5] = [60000.0, -1.0, 3.0, 0.5, 2.0]
    cache, scales, c_out, st = run_append(E, E, B, x, 16.0 * np.eye(E), "i4", "f32")
    exact = (16.0 * x).astype(np.float32)
    assert np.array_equal(c_out, exact)
    codes, s16, ovf = qr.quantize(exact, 4, 128)
    assert ovf[0, 0] and st & q.QSVD_STATUS_SCALE_SAT
    rows, _ = expected_rows(exact, "i4", 128)
    assert np.array_equal(cache[0, 0], rows[0])
    assert np.array_equal(scales[0, 0].view(np.uint16), s16[0].view(np.uint16))


@pytest.mark.parametrize("cache_dtype", ["i4", "i8", "f16"])
def test_dyadic_projection_bit_exact_llava_shapes(cuda_ok, cache_dtype):
    """E = 4096, r = 768, B = 32 (the int4 configuration's append): integer
    activations and weights on a 1/8 grid make x W^d exact in float32."""
    B, E, r = 32, 4096, 768
    g = np.random.default_rng(7)
    x = g.integers(-3, 4, size=(B, E)).astype(np.float32)
    wd = g.integers(-16, 17, size=(E, r)).astype(np.float64) / 8.0
    exact = x.astype(np.float64) @ wd
    assert np.max(np.abs(exact)) < 2 ** 20
    cache, scales, c_out, st = run_append(E, r, B, x, wd, cache_dtype, "f16", max_len=40)
    assert np.array_equal(c_out.astype(np.float64), exact)
    rows, s16 = expected_rows(exact.astype(np.float32), cache_dtype, 128)
    for b in range(B):
        assert np.array_equal(cache[b, b % 40], rows[b])
        if s16 is not None:
            assert np.array_equal(scales[b, b % 40].view(np.uint16), s16[b].view(np.uint16))


def test_online_h2_rotation(cuda_ok):
    """c = H2 (x W^d) with H2 = H_128 (x) Q3 (r = 384), against the oracle."""
    w = synthetic.SHRUNK[3]
    B, E, r = 3, w.E, w.r
    g = np.random.default_rng(5)
    x = np.asarray((g.standard_normal((B, E))).astype(np.float16), np.float32)
    wd = g.standard_normal((E, r)) / np.sqrt(E)
    wd16 = oi.from_device_dtype(oi.to_device_dtype(wd, "f16"), "f16")
    q3 = synthetic.dct3()
    cache, scales, c_out, st = run_append(E, r, B, x, wd16, "i4", "f16", h2=True,
                                          h2_q=q3.astype(np.float32), h2_m=3)
    h2 = ref.h2_matrix(128, q3.astype(np.float32).astype(np.float64))
    want = (x.astype(np.float64) @ wd16) @ h2.T
    assert np.max(np.abs(c_out - want)) <= 1e-5 * np.max(np.abs(want))
    # The quantise/pack step is bit-exact on the latent the kernel reports:
    # the codes and the fp16 scales of quantize(c_out) are the stored bytes.
    codes_w, s16_w, _ = qr.quantize(c_out.astype(np.float32), 4, 128)
    got_codes = np.stack([qr.unpack_int4(cache[b, b][None, :])[0] for b in range(B)])
    assert np.array_equal(got_codes, codes_w.reshape(got_codes.shape))
    got_s = np.stack([scales[b, b] for b in range(B)])
    assert np.array_equal(got_s.view(np.uint16), s16_w.astype(np.float16).reshape(got_s.shape).view(np.uint16))
    # and the packed row is the oracle's packing of those codes
    want_rows = qr.pack_int4(codes_w)
    for b in range(B):
        assert np.array_equal(cache[b, b], want_rows[b])


def test_position_out_of_range(cuda_ok):
    B, E = 2, 256
    x = np.ones((B, E), np.float32)
    cache, scales, c_out, st = run_append(E, E, B, x, np.eye(E), "i8", "f16",
                                          max_len=4, pos=[4, -1])
    assert st & q.QSVD_STATUS_POS_OOB
    assert not cache.any()
