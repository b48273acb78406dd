"""Parity of the per-head latent decode (qsvd_decode_attn_per_head; WSVD
digest, Method §3.1, §3.4) with the oracle (``oracle.wsvd_ref``).

Both sides get the same rounded inputs: per-head factors B_{Kh}, B_{Vh} in the
weight type, key and value latents in the cache type, the float32 query.
The kernels compute in float32 throughout, so the bar is that of the
float32 decode tests: max |o_gpu - o_ref| / rms(o_ref) <= 1e-4.  Rows past
each sequence's length hold a large value, so reading them shows.
"""
import numpy as np
import pytest
import torch

import rank_joint_qkv_b200 as q
import synthetic
from oracle import inputs as oi
from oracle import wsvd_ref as wr
from tests.gpu_util import rel_err

pytestmark = pytest.mark.gpu
TOL = 1e-4
PAD = 3.0e4


def _case(E, H, r, lengths, cache, weight):
    w = synthetic.replace(synthetic.SHRUNK[1], E=E, H=H, d_h=E // H, r=r, B=len(lengths), L=max(lengths))
    wq, wk, wv = synthetic.qkv_weights(w)
    fk = wr.per_head_factors(wk, H, r)
    fv = wr.per_head_factors(wv, H, r)
    rnd = lambda m, dt: oi.from_device_dtype(oi.to_device_dtype(m, dt), dt)
    fk = [(a, rnd(b, weight)) for a, b in fk]
    fv = [(a, rnd(b, weight)) for a, b in fv]
    max_len = max(max(lengths), 1) + 7
    d_h = E // H
    ck = np.full((len(lengths), H, max_len, r), PAD)
    cv = np.full((len(lengths), H, max_len, r), PAD)
    qv = np.zeros((len(lengths), E), np.float32)
    for b, n in enumerate(lengths):
        x = synthetic.sequence_activations(w, b, max(n, 1)).astype(np.float64)
        ck[b, :, :n] = rnd(wr.per_head_latents(x[:n], fk), cache)
        cv[b, :, :n] = rnd(wr.per_head_latents(x[:n], fv), cache)
        qv[b] = (x[max(n, 1) - 1] @ wq.astype(np.float64)).astype(np.float32)
    want = wr.decode_absorbed([ck[b] for b in range(len(lengths))], [cv[b] for b in range(len(lengths))],
                              np.asarray(lengths), qv.astype(np.float64), fk, fv)
    dims = q.make_dims(E, H, d_h, r, len(lengths), max_len, cache=cache, weight=weight)
    dev = dict(
        bk=oi.as_torch(oi.to_device_dtype(np.stack([b for _, b in fk]), weight), weight).cuda(),
        bv=oi.as_torch(oi.to_device_dtype(np.stack([b for _, b in fv]), weight), weight).cuda(),
        ck=oi.as_torch(oi.to_device_dtype(ck, cache), cache).cuda(),
        cv=oi.as_torch(oi.to_device_dtype(cv, cache), cache).cuda(),
        q=torch.from_numpy(qv).cuda(),
        lengths=torch.tensor(lengths, dtype=torch.int32).cuda())
    return dims, dev, want


def _run(dims, dev, out_dtype=torch.float32):
    out = torch.full((dims.batch, dims.E), float("nan"), dtype=out_dtype, device="cuda")
    ws = q.qsvd_decode_attn_per_head(dims, dev["bk"], dev["bv"], dev["q"], dev["ck"], dev["cv"],
                                     dev["lengths"], out)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), int(ws[:4].view(torch.int32).item())


@pytest.mark.parametrize("E,H,r,lengths,cache,weight", [
    (512, 4, 64, [300, 1, 513], "f16", "f16"),      # several chunks, a one-token sequence, a ragged tail
    (512, 4, 32, [256, 257], "bf16", "bf16"),      # chunk boundary exactly and one past
    (512, 4, 96, [700], "f32", "f16"),             # r not dividing the thread count
    (1024, 8, 128, [1000, 40], "f16", "bf16"),
    (512, 2, 256, [600, 3], "f16", "f16"),         # r above the thread count
])
def test_matches_oracle(cuda_ok, E, H, r, lengths, cache, weight):
    dims, dev, want = _case(E, H, r, lengths, cache, weight)
    got, status = _run(dims, dev)
    assert status == 0
    assert rel_err(got, want) <= TOL


def test_empty_and_clamped_lengths(cuda_ok):
    """len 0 gives a zero row; a length beyond max_len is clamped to it and
    flagged; a negative one reads nothing and is flagged."""
    dims, dev, _ = _case(512, 4, 64, [200, 0, 100], "f16", "f16")   # max_len 207
    dev["lengths"] = torch.tensor([200, 0, 10 ** 6], dtype=torch.int32, device="cuda")
    got, status = _run(dims, dev)
    assert status & q.QSVD_STATUS_LEN_CLAMPED
    assert np.all(got[1] == 0.0)
    assert np.all(np.isfinite(got))
    dev["lengths"] = torch.tensor([200, -3, 200], dtype=torch.int32, device="cuda")
    got, status = _run(dims, dev)
    assert status & q.QSVD_STATUS_LEN_CLAMPED and np.all(got[1] == 0.0)


def test_out_dtypes_round_the_float32_result(cuda_ok):
    dims, dev, _ = _case(512, 4, 64, [300, 77], "f16", "f16")
    ref32, _ = _run(dims, dev)
    for dt, td in (("f16", torch.float16), ("bf16", torch.bfloat16)):
        dims.out_dtype = q.DTYPE_CODE[dt]
        got, _ = _run(dims, dev, td)
        want = oi.from_device_dtype(oi.to_device_dtype(ref32, dt), dt)
        assert np.array_equal(got, want.astype(np.float32))
