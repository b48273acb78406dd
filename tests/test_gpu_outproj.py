"""Parity of the output projection applied by the combine: CHAIN (V-up, then
y = o W_O) and FOLD (y = sum_h z_h F_h, F_h = W^u_{v,h} W_{O,h} formed once at
prepare time; WSVD digest, Method, fused kernel §3.4).

Oracle: the materialised decode of the case times W_O (chain), and the
per-head latents times the fold rounded to the weight type (fold: the stored
F is defined as the float32 fold rounded once).  Bar as for the tensor-core
decode: max |y_gpu - y_ref| / rms(y_ref) <= 2e-3.  The stored F itself is
compared with the exact fold element by element: within the float32
accumulation bound d_h 2^-24 sum_i |W^u_v[j][i]| |W_O[i][n]| plus one
rounding to the 16-bit type, and equal to the oracle's rounded fold on all
but 0.1% of the entries (float32 and float64 sums can round to neighbouring
values; an entry with heavy cancellation can differ by many units in its
last place while its absolute error stays within the bound).
"""
import numpy as np
import pytest
import torch

import rank_joint_qkv_b200 as q
import synthetic
from oracle import inputs as oi
from oracle import qsvd_ref as ref
from tests.gpu_util import GpuCase, dev_tensor, rel_err

pytestmark = pytest.mark.gpu
TOL = 2e-3
TC = q.QSVD_KERNEL_TCGEN05

_CASES = {}


def case(key):
    if key not in _CASES:
        base = synthetic.SHRUNK[1]   # E=512, H=4, r=256, B=3, L=300 (ragged tail)
        w = {
            "f16": base,
            "bf16": synthetic.replace(base, cache="bf16", weight="bf16"),
            "h32": synthetic.replace(base, E=4096, H=32, r=384, B=2, L=520),
            "i4": synthetic.replace(synthetic.SHRUNK[3], r=256, h2_n=0, h2_m=0),
            "rope": synthetic.SHRUNK[2],
        }[key]
        if w.E > 1024:
            wuq, wuk, wuv = (a.astype(np.float64) for a in synthetic.direct_up_weights_np(w))
            wd = synthetic.direct_down_weight_np(w).astype(np.float64)
            c = oi.build_case(w, factors_override=(0.5, (wd, wuq, wuk, wuv), None))
        else:
            c = oi.build_case(w)
        g = np.random.default_rng(77)
        wo_dev = oi.to_device_dtype(g.standard_normal((w.E, w.E)) / np.sqrt(w.E), w.weight)
        _CASES[key] = (c, wo_dev, oi.from_device_dtype(wo_dev, w.weight))
    return _CASES[key]


def gpu_case(c, wo_dev, mode, out="f32"):
    g = GpuCase(c, kernel=TC, out=out)
    g.dims.out_proj = q.OUT_PROJ_CODE[mode]
    g.packed = q.qsvd_prepare_weights(g.dims, g.wd, g.wuq, g.wuk, g.wuv)
    q.qsvd_prepare_out_proj(g.dims, dev_tensor(wo_dev, c.w.weight), g.packed)
    return g


def stored_fold(g, c):
    """F as laid out in the packed buffer (the last section)."""
    w = c.w
    n = w.H * w.r * w.E * 2
    total = g.packed.numel()
    start = total - (n + 255) // 256 * 256
    raw = g.packed[start:start + n].cpu().numpy()
    dt = np.float16 if w.weight == "f16" else np.uint16
    return raw.view(dt).reshape(w.H * w.r, w.E)


def rounded_fold(c, wo_v):
    f = ref.fold_value_output(c.wuv, wo_v, c.w.H)
    return oi.to_device_dtype(f, c.w.weight)


def check_stored_fold(f_dev, c, wo_v):
    w = c.w
    exact = ref.fold_value_output(c.wuv, wo_v, w.H)
    absprod = ref.fold_value_output(np.abs(c.wuv), np.abs(wo_v), w.H)
    acc = w.d_h * 2.0 ** -24 * absprod            # float32 accumulation bound
    u = 2.0 ** -11 if w.weight == "f16" else 2.0 ** -8
    bound = u * (np.abs(exact) + acc) + acc + 2.0 ** -25
    got = oi.from_device_dtype(f_dev, w.weight)
    assert np.all(np.abs(got - exact) <= bound), np.max(np.abs(got - exact) / bound)
    same = got == oi.from_device_dtype(oi.to_device_dtype(exact, w.weight), w.weight)
    assert np.mean(~same) <= 1e-3, np.mean(~same)


@pytest.mark.parametrize("key", ["f16", "bf16", "h32", "i4", "rope"])
def test_chain_matches_oracle(cuda_ok, key):
    c, wo_dev, wo_v = case(key)
    g = gpu_case(c, wo_dev, "chain")
    got, _ = g.decode()
    want = ref.output_projection(c.reference(), wo_v)
    assert rel_err(got, want) <= TOL


@pytest.mark.parametrize("key", ["f16", "bf16", "h32", "i4", "rope"])
def test_fold_matches_oracle(cuda_ok, key):
    c, wo_dev, wo_v = case(key)
    w = c.w
    g = gpu_case(c, wo_dev, "fold")
    check_stored_fold(stored_fold(g, c), c, wo_v)
    f_ref = rounded_fold(c, wo_v)
    got, _ = g.decode()
    z = ref.decode_absorbed_latents(c.caches, c.lengths, c.cnew.astype(np.float64), c.wuq, c.wuk, w.H,
                                    rope_base=w.rope_base if w.rope else None)
    want = ref.decode_folded(z, oi.from_device_dtype(f_ref, w.weight))
    assert rel_err(got, want) <= TOL
    # against the exact projected attention the fold's own rounding adds on
    # (measured by the oracle: rounded fold vs unrounded)
    exact = ref.output_projection(c.reference(), wo_v)
    rms = np.sqrt(np.mean(exact ** 2))
    assert np.max(np.abs(got - exact)) <= TOL * np.sqrt(np.mean(want ** 2)) + \
        np.max(np.abs(want - exact)) + 1e-12 * rms


@pytest.mark.parametrize("mode", ["chain", "fold"])
def test_phases_separately_bit_identical(cuda_ok, mode):
    c, wo_dev, _ = case("f16")
    g = gpu_case(c, wo_dev, mode, out="f16")
    one, _ = g.decode()
    sep, _ = g.decode(phases_separately=True)
    assert np.array_equal(one.view(np.uint32), sep.view(np.uint32))
    assert np.all(np.isfinite(one))


def test_chain_with_identity_is_plain_decode(cuda_ok):
    """W_O = I: the chain's output is the plain decode's to the fp32
    hi/lo split of o (two 16-bit parts carry ~16 bits)."""
    c, _, _ = case("f16")
    w = c.w
    eye = oi.to_device_dtype(np.eye(w.E), w.weight)
    plain, _ = GpuCase(c, kernel=TC).decode()
    got, _ = gpu_case(c, eye, "chain").decode()
    assert rel_err(got, plain) <= 1e-4
