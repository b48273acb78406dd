"""Decode parity: CUDA path vs the fp64 oracle on identical seeded inputs.

Bar (stated for the decode path): max |o_gpu - o_ref| / rms(o_ref) <= 2e-3
for 16-bit and quantised latents (quantised: against the oracle on the same
dequantised values); 1e-4 for float32 latents, whose kernels never round
below float32.
"""
import numpy as np
import pytest
import torch

import rank_joint_qkv_b200 as q
import synthetic
from oracle import inputs as oi
from oracle import qsvd_ref as ref
from tests.gpu_util import GpuCase, rel_err, DEV

pytestmark = pytest.mark.gpu

TOL = 2e-3
TOL_F32 = 1e-4

_CASES = {}


def case_for(key):
    if key not in _CASES:
        if key == "cfg0":
            w = synthetic.CONFIGS[0]
        elif key == "s3-i8":
            w = synthetic.replace(synthetic.SHRUNK[3], cache="i8", name="shrunk-int8-h2")
        elif key == "s1-f32w":
            w = synthetic.replace(synthetic.SHRUNK[1], weight="f32", cache="f32")
        elif key == "s1-bf16":
            w = synthetic.replace(synthetic.SHRUNK[1], weight="bf16", cache="bf16")
        elif key == "s1-dh96":   # 16-bit weights, d_h not a multiple of 64: one-kernel combine
            w = synthetic.replace(synthetic.SHRUNK[1], E=384, H=4, d_h=96)
        else:
            w = synthetic.SHRUNK[int(key[1])]
        _CASES[key] = oi.build_case(w)
    return _CASES[key]


ALL = ["cfg0", "s1", "s1-bf16", "s1-f32w", "s1-dh96", "s2", "s3", "s3-i8", "s4"]


@pytest.mark.parametrize("key", ALL)
def test_decode_matches_oracle(cuda_ok, key):
    case = case_for(key)
    g = GpuCase(case)
    got, ws = g.decode()
    want = case.reference()
    tol = TOL_F32 if case.w.cache == "f32" else TOL
    err = rel_err(got, want)
    assert err <= tol, f"{key}: rel err {err:.3e}"
    assert q.status_word(ws) == 0


@pytest.mark.parametrize("key", ["s1", "s3", "s4"])
@pytest.mark.parametrize("splits", [1, 2, 5, 1000])
def test_split_count_invariance(cuda_ok, key, splits):
    """Any split count gives the same attention (log-sum-exp merge).  The
    split kernel here is exact fp32; the combine's V-up takes the merged
    latent into the tensor cores as two 16-bit parts (22 significant bits),
    so split counts, which round the merged latent differently, agree to a
    few units of 2^-22 per term summed over r."""
    case = case_for(key)
    g = GpuCase(case)
    base, _ = g.decode(num_splits=1)
    got, _ = g.decode(num_splits=splits)
    assert rel_err(got, base) <= 4e-5
    assert rel_err(got, case.reference()) <= (TOL_F32 if case.w.cache == "f32" else TOL)


@pytest.mark.parametrize("key", ["s1", "s2"])
def test_phases_run_separately(cuda_ok, key):
    case = case_for(key)
    g = GpuCase(case)
    a, _ = g.decode(num_splits=3)
    b, _ = g.decode(num_splits=3, phases_separately=True)
    assert np.array_equal(a, b)


@pytest.mark.parametrize("key", ["s1", "s2"])
def test_query_given_directly(cuda_ok, key):
    """qin as the E-wide query (q = c_new W^u_q computed by the oracle)."""
    case = case_for(key)
    g = GpuCase(case)
    qv = (case.cnew.astype(np.float64) @ case.wuq).astype(np.float32)
    got, _ = g.decode(qin=torch.from_numpy(qv).to(DEV), qin_is_latent=False)
    rb = case.w.rope_base if case.w.rope else None
    want = ref.decode_materialized(case.caches, case.lengths, qv.astype(np.float64), case.wuq,
                                   case.wuk, case.wuv, case.w.H, qin_is_latent=False,
                                   rope_base=rb)
    assert rel_err(got, want) <= TOL


@pytest.mark.parametrize("key", ["s1", "s2", "s3"])
@pytest.mark.parametrize("lens", [[0, 1, 2], [127, 128, 129], [1, 0, 300], [255, 256, 257]])
def test_edge_lengths(cuda_ok, key, lens):
    """Empty, single-token and tile-boundary lengths; len 0 gives zeros."""
    w0 = synthetic.SHRUNK[int(key[1])]
    w = synthetic.replace(w0, B=len(lens), ragged=None, L=max(lens))
    case = oi.build_case(w, lengths=np.array(lens, np.int32))
    g = GpuCase(case)
    got, ws = g.decode(num_splits=2)
    want = case.reference()
    for b, n in enumerate(lens):
        if n == 0:
            assert np.all(got[b] == 0.0)
    assert rel_err(got, want) <= TOL
    assert q.status_word(ws) == 0


def test_padding_rows_never_read(cuda_ok):
    """Rows at or past each length hold NaN: nothing may leak."""
    case = oi.build_case(synthetic.SHRUNK[1])
    g = GpuCase(case)
    for b, n in enumerate(case.lengths):
        g.cache[b, int(n):] = float("nan")
    got, _ = g.decode(num_splits=4)
    assert np.all(np.isfinite(got))
    assert rel_err(got, case.reference()) <= TOL


def test_lengths_out_of_range_are_clamped_and_flagged(cuda_ok):
    case = case_for("s1")
    g = GpuCase(case)
    lens = torch.tensor([case.max_len + 50, -3, 10], dtype=torch.int32, device=DEV)
    got, ws = g.decode(lengths=lens)
    assert q.status_word(ws) & q.QSVD_STATUS_LEN_CLAMPED
    clamped = np.array([case.max_len, 0, 10])
    # rows up to max_len hold the pad value; compare to the oracle on exactly that
    caches = [oi.from_device_dtype(case.cache_dev[b], case.w.cache) for b in range(3)]
    want = ref.decode_materialized(caches, clamped, case.cnew.astype(np.float64), case.wuq,
                                   case.wuk, case.wuv, case.w.H)
    assert np.all(got[1] == 0.0)
    assert rel_err(got[[0, 2]], want[[0, 2]]) <= TOL


@pytest.mark.parametrize("out", ["f16", "bf16"])
def test_output_dtypes(cuda_ok, out):
    case = case_for("s1")
    g = GpuCase(case, out=out)
    got, _ = g.decode()
    want = case.reference()
    rms = np.sqrt(np.mean(want ** 2))
    ulp = 2.0 ** (-8 if out == "bf16" else -11)      # half an ulp of the output type
    assert np.all(np.abs(got - want) <= TOL * rms + ulp * np.abs(want))
