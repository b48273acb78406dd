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
    dev["host"] = ([ck[b] for b in range(len(lengths))], [cv[b] for b in range(len(lengths))], qv, fk, fv)
    return dims, dev, want


def _run(dims, dev, out_dtype=torch.float32, layout=q.QSVD_PER_HEAD_HEAD_MAJOR):
    out = torch.full((dims.batch, dims.E), float("nan"), dtype=out_dtype, device="cuda")
    ck, cv = dev["ck"], dev["cv"]
    if layout == q.QSVD_PER_HEAD_TOKEN_MAJOR:   # B x H x L x r -> B x L x H x r
        ck, cv = ck.transpose(1, 2).contiguous(), cv.transpose(1, 2).contiguous()
    ws = q.qsvd_decode_attn_per_head(dims, dev["bk"], dev["bv"], dev["q"], ck, cv,
                                     dev["lengths"], out, layout=layout)
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
    # the token-major layout reads the same rows: the same bits
    got_tm, status = _run(dims, dev, layout=q.QSVD_PER_HEAD_TOKEN_MAJOR)
    assert status == 0 and np.array_equal(got_tm, got)


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


def test_latents_from_prefill(cuda_ok):
    """Per-head key and value latents written by qsvd_prefill_latent (W^d =
    [A_1 .. A_H], rank H r, one cache row per token holding every head) and
    read by the per-head decode in the token-major layout.

    The prefill sums in float32 in the tensor cores' order, so a latent that
    sits next to an fp16 rounding boundary may round the other way than the
    float64 product does.  Two checks therefore: (1) each stored row is the
    fp16 rounding of the float32 latent the prefill reports, and that latent
    is within the prefill's accumulation bound of the float64 product;
    (2) the decode is compared with the oracle run on the stored bytes
    themselves (the same-input bar of the per-head path)."""
    E, H, r, lengths = 512, 4, 64, [300, 1, 513]
    d_h = E // H
    w = synthetic.replace(synthetic.SHRUNK[1], E=E, H=H, d_h=d_h, r=r, B=len(lengths), L=max(lengths))
    wq, wk, wv = synthetic.qkv_weights(w)
    rnd = lambda m: oi.from_device_dtype(oi.to_device_dtype(m, "f16"), "f16")
    fk = [(rnd(a), rnd(b)) for a, b in wr.per_head_factors(wk, H, r)]
    fv = [(rnd(a), rnd(b)) for a, b in wr.per_head_factors(wv, H, r)]
    max_len = max(lengths) + 5
    xs = [rnd(synthetic.sequence_activations(w, b, n)) for b, n in enumerate(lengths)]
    qv = np.stack([(x[-1] @ wq.astype(np.float64)).astype(np.float32) for x in xs])

    R = H * r
    n_tok = sum(lengths)
    pdims = q.make_dims(E, H, d_h, R, len(lengths), max_len, cache="f16", weight="f16")
    x_all = torch.from_numpy(np.concatenate(xs).astype(np.float16)).cuda()
    rows_np = np.concatenate([b * max_len + np.arange(n) for b, n in enumerate(lengths)])
    rows = torch.from_numpy(rows_np.astype(np.int32)).cuda()
    zeros = torch.zeros((R, E), dtype=torch.float16, device="cuda")
    caches = []
    for fac in (fk, fv):
        a_all_np = np.concatenate([a for a, _ in fac], axis=1)
        a_all = torch.from_numpy(a_all_np.astype(np.float16)).cuda()
        packed = q.qsvd_prepare_weights(pdims, a_all, zeros, zeros, zeros)
        cache = torch.full((len(lengths), max_len, R), PAD, dtype=torch.float16, device="cuda")
        c32 = torch.empty((n_tok, R), dtype=torch.float32, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        q.qsvd_prefill_latent(pdims, packed, x_all, rows, cache, c_out=c32, status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        # (1) the stored rows are exactly the fp16 rounding of the reported latent
        stored = cache.view(-1, R)[rows.long()].cpu().numpy()
        c32_np = c32.cpu().numpy()
        assert np.array_equal(stored, c32_np.astype(np.float16))
        exact = np.concatenate(xs) @ a_all_np
        assert np.max(np.abs(c32_np - exact)) <= 1e-5 * np.sqrt(np.mean(exact ** 2))
        caches.append(cache)
    # (2) the oracle on the bytes the prefill stored, as H x len x r per sequence
    host = [c.cpu().numpy().astype(np.float64) for c in caches]
    ck = [host[0][b, :n].reshape(n, H, r).transpose(1, 0, 2) for b, n in enumerate(lengths)]
    cv = [host[1][b, :n].reshape(n, H, r).transpose(1, 0, 2) for b, n in enumerate(lengths)]
    want = wr.decode_absorbed(ck, cv, np.asarray(lengths), qv.astype(np.float64), fk, fv)

    dims = q.make_dims(E, H, d_h, r, len(lengths), max_len, cache="f16", weight="f16")
    bk = torch.from_numpy(np.stack([b for _, b in fk]).astype(np.float16)).cuda()
    bv = torch.from_numpy(np.stack([b for _, b in fv]).astype(np.float16)).cuda()
    out = torch.full((len(lengths), E), float("nan"), dtype=torch.float32, device="cuda")
    ws = q.qsvd_decode_attn_per_head(dims, bk, bv, torch.from_numpy(qv).cuda(), caches[0], caches[1],
                                     torch.tensor(lengths, dtype=torch.int32, device="cuda"), out,
                                     layout=q.QSVD_PER_HEAD_TOKEN_MAJOR)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0
    assert rel_err(out.cpu().numpy(), want) <= TOL


@pytest.mark.parametrize("weight", ["f16", "bf16"])
def test_value_factor_folded_into_output_projection(cuda_ok, weight):
    """B_{Vh} folded into W_O on the GPU (WSVD digest, Method, fused kernel
    §3.4): F = [B_{Vh} W_{O,h}]_h against the oracle's fold (float32
    accumulation over d_h terms plus one rounding to the weight type), and
    the folded decode y = z F against the oracle's merged latents times the
    stored F (float32 arithmetic: the per-head bar)."""
    E, H, r, lengths = 512, 4, 64, [300, 1, 130]
    d_h = E // H
    dims, dev, _ = _case(E, H, r, lengths, weight, weight)
    g = np.random.default_rng(3)
    wo = oi.from_device_dtype(oi.to_device_dtype(g.standard_normal((E, E)) / np.sqrt(E), weight), weight)
    wo_t = oi.as_torch(oi.to_device_dtype(wo, weight), weight).cuda()
    f = q.qsvd_prepare_per_head_fold(dims, dev["bv"], wo_t)
    torch.cuda.synchronize()
    f_np = f.float().cpu().numpy().astype(np.float64)
    ck, cv, qv, fk, fv = dev["host"]
    f64 = wr.fold_values(fv, wo)
    acc = np.concatenate([np.abs(b) @ np.abs(wo[h * d_h:(h + 1) * d_h]) for h, (_, b) in enumerate(fv)])
    ulp = 2.0 ** (-11 if weight == "f16" else -8)
    assert np.all(np.abs(f_np - f64) <= ulp * np.abs(f64) + d_h * 2.0 ** -23 * acc + 1e-30)
    dims.out_proj = q.OUT_PROJ_CODE["fold"]
    out = torch.full((dims.batch, E), float("nan"), dtype=torch.float32, device="cuda")
    ws = q.qsvd_decode_attn_per_head(dims, dev["bk"], f, dev["q"], dev["ck"], dev["cv"], dev["lengths"], out)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0
    z = wr.decode_latents(ck, cv, np.asarray(lengths), qv.astype(np.float64), fk)
    want = z.reshape(len(lengths), -1) @ f_np
    assert rel_err(out.cpu().numpy(), want) <= TOL


@pytest.mark.parametrize("r,dt,layout", [(64, "f16", q.QSVD_PER_HEAD_HEAD_MAJOR),
                                         (128, "bf16", q.QSVD_PER_HEAD_TOKEN_MAJOR),
                                         (64, "f16", q.QSVD_PER_HEAD_TOKEN_MAJOR)])
def test_rotary_keys_rebuilt_on_tensor_cores(cuda_ok, r, dt, layout):
    """Rotary mode (WSVD digest, Method §3.4: keys rebuilt from the per-head
    latent tile and rotated before the scores): K_h = C_{Kh} B_{Kh} on
    tcgen05, rotated at each position, the query at len - 1; against the
    oracle's rebuilt-key decode.  Bar: 2e-3 (16-bit operands, float32
    tensor-core accumulation)."""
    E, H, lengths = 512, 4, [300, 1, 513]
    dims, dev, _ = _case(E, H, r, lengths, dt, dt)
    ck, cv, qv, fk, fv = dev["host"]
    want = wr.decode(ck, cv, np.asarray(lengths), qv.astype(np.float64), fk, fv, rope_base=10000.0)
    dims.rope, dims.rope_base = 1, 10000.0
    got, status = _run(dims, dev, layout=layout)
    assert status == 0
    assert rel_err(got, want) <= 2e-3
