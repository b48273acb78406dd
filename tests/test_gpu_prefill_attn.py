"""Prefill attention (qsvd_prefill_attention) against the oracle's causal
attention over a prompt's latent rows (QSVD digest, Method, Step 1: queries,
keys and values rebuilt from the buffered latent), with and without rotary
embedding, fp16 and bf16, ragged prompts that span several 128-query tiles,
a one-token prompt and an empty one."""
import numpy as np
import pytest
import torch

import rank_joint_qkv_b200 as q
import synthetic
from oracle import inputs as oi
from oracle import qsvd_ref as ref
from tests.gpu_util import GpuCase, rel_err

pytestmark = pytest.mark.gpu
TOL = 2e-3


@pytest.mark.parametrize("key,dt,rope,lengths", [
    (1, "f16", False, [300, 1, 129]),
    (1, "bf16", False, [257, 128, 0]),
    (2, "bf16", True, [290, 64]),
    (2, "f16", True, [200, 290, 5]),
])
def test_prefill_attention_matches_oracle(cuda_ok, key, dt, rope, lengths):
    w = synthetic.replace(synthetic.SHRUNK[key], cache=dt, weight=dt, rope=rope, B=len(lengths),
                          L=max(lengths), ragged=None)
    case = oi.build_case(w, lengths=np.asarray(lengths, np.int32))
    g = GpuCase(case, kernel=q.QSVD_KERNEL_AUTO)
    B, max_len, E = w.B, case.max_len, w.E
    out = torch.full((B, max_len, E), float("nan"), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    q.qsvd_prefill_attention(g.dims, g.packed, g.cache, g.lengths, out, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    got = out.cpu().numpy()
    rb = w.rope_base if rope else None
    for b, n in enumerate(lengths):
        assert np.all(np.isnan(got[b, n:]))            # rows past the prompt are left alone
        if n == 0:
            continue
        want = ref.prefill_attention(case.caches[b][:n], case.wuq, case.wuk, case.wuv, w.H, rope_base=rb)
        assert rel_err(got[b, :n], want) <= TOL, f"prompt {b}"


def test_prefill_attention_output_types_round_the_float32_result(cuda_ok):
    w = synthetic.replace(synthetic.SHRUNK[1], B=2, L=200, ragged=None)
    case = oi.build_case(w, lengths=np.asarray([200, 77], np.int32))
    g = GpuCase(case, kernel=q.QSVD_KERNEL_AUTO)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ref32 = torch.zeros((2, case.max_len, w.E), dtype=torch.float32, device="cuda")
    q.qsvd_prefill_attention(g.dims, g.packed, g.cache, g.lengths, ref32, st)
    for name, td in (("f16", torch.float16), ("bf16", torch.bfloat16)):
        g.dims.out_dtype = q.DTYPE_CODE[name]
        o = torch.zeros((2, case.max_len, w.E), dtype=td, device="cuda")
        q.qsvd_prefill_attention(g.dims, g.packed, g.cache, g.lengths, o, st)
        torch.cuda.synchronize()
        assert torch.equal(o[0, :200], ref32[0, :200].to(td)) and torch.equal(o[1, :77], ref32[1, :77].to(td))
    assert int(st.item()) == 0
