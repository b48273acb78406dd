"""Full-size parity in the benchmark's launch configuration, on sampled
sequences the oracle can compute one by one.

The benchmark's device inputs (bench.bench_inputs: seeded synthetic latent
rows and weights) are decoded with the benchmark's split count and kernel;
the oracle rebuilds keys and values for two sampled sequences in float64.
"""
import numpy as np
import pytest
import torch

import bench
import rank_joint_qkv_b200 as q
import synthetic
from oracle import qsvd_ref as ref
from oracle import quant_ref as qr
from tests.gpu_util import rel_err

pytestmark = pytest.mark.gpu


def _latent_rows(inp, w, b, n):
    """Sequence b's first n latent rows as float64: 16-bit values as stored,
    quantised codes dequantised exactly (code x fp16 group scale)."""
    if w.cache in ("f32", "f16", "bf16"):
        return inp["cache"][b, :n].float().cpu().numpy().astype(np.float64)
    raw = inp["cache"][b, :n].cpu().numpy()
    codes = qr.unpack_int4(raw) if w.cache == "i4" else raw.view(np.int8)
    sc = inp["scales"][b, :n].cpu().numpy()
    return qr.dequantize(codes, sc, w.group).astype(np.float64)


def _run(cfg, kernel, cache=None):
    dev = "cuda"
    inp = bench.bench_inputs(cfg, dev, cache=cache)
    w, lens, max_len = inp["w"], inp["lens"], inp["max_len"]
    kern = {"auto": q.QSVD_KERNEL_AUTO, "simt": q.QSVD_KERNEL_SIMT,
            "tcgen05": q.QSVD_KERNEL_TCGEN05}[kernel]
    dims = q.make_dims(w.E, w.H, w.d_h, w.r, w.B, max_len, cache=w.cache, weight=w.weight,
                       group=w.group, rope=w.rope, rope_base=w.rope_base, kernel=kern)
    packed = q.qsvd_prepare_weights(dims, inp["wd"], inp["wuq"], inp["wuk"], inp["wuv"])
    cnew = synthetic.direct_new_latent_np(w)
    out = torch.empty((w.B, w.E), dtype=torch.float32, device=dev)
    lens_dev = torch.from_numpy(lens).to(dev)
    ws = q.qsvd_decode_attn(dims, packed, torch.from_numpy(cnew).to(dev), True, inp["cache"],
                            inp["scales"], lens_dev, out)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0
    wuq, wuk, wuv = (t.float().cpu().numpy().astype(np.float64)
                     for t in (inp["wuq"], inp["wuk"], inp["wuv"]))
    return inp, w, lens, cnew, out.cpu().numpy(), (wuq, wuk, wuv)


# cfg 1: fp16 absorbed; cfg 3: int4 + H2 workload, and the same shapes with
# an int8 latent (quantised latents on the tensor cores); cfg 2 / 4: bf16
# rotary (keys rebuilt on the tensor cores, then the given-scores pass).
# Every sampled sequence is compared whole (all heads); cfg 4's longest
# sequence is compared head by head in the next test.
@pytest.mark.parametrize("cfg,cache", [(1, None), (3, None), (3, "i8"), (2, None), (4, None)])
def test_fullsize_sampled(cuda_ok, cfg, cache):
    inp, w, lens, cnew, got, (wuq, wuk, wuv) = _run(cfg, "auto", cache)
    rb = w.rope_base if w.rope else None
    picks = (0, w.B - 1) if cfg != 4 else tuple(int(i) for i in np.argsort(lens)[:2])
    for b in picks:
        n = int(lens[b])
        c = _latent_rows(inp, w, b, n)
        want = ref.decode_materialized([c], [n], cnew[b:b + 1].astype(np.float64), wuq, wuk,
                                       wuv, w.H, rope_base=rb)
        assert rel_err(got[b:b + 1], want) <= 2e-3


def test_fullsize_longest_rotary_sequence(cuda_ok):
    """The LLaVA-13B rotary workload's longest sequence (up to 32,768 tokens):
    rotary angles at positions past 16k, where a float32 angle would be off
    by ~2^-9 rad.  Heads are independent (head h owns columns h d_h ..), so
    the oracle runs one head at a time on that head's columns of W^u and the
    comparison covers a spread of heads, keeping the float64 keys and values
    of one head (32k x 128) small."""
    inp, w, lens, cnew, got, (wuq, wuk, wuv) = _run(4, "auto")
    b = int(np.argmax(lens))
    n = int(lens[b])
    assert n > 30000
    c = _latent_rows(inp, w, b, n)
    heads = (0, 7, 19, 26, w.H - 1)
    d = w.d_h
    want = np.concatenate([
        ref.decode_materialized([c], [n], cnew[b:b + 1].astype(np.float64),
                                wuq[:, h * d:(h + 1) * d], wuk[:, h * d:(h + 1) * d],
                                wuv[:, h * d:(h + 1) * d], 1, rope_base=w.rope_base)
        for h in heads], axis=1)
    sel = np.concatenate([np.arange(h * d, (h + 1) * d) for h in heads])
    assert rel_err(got[b:b + 1, sel], want) <= 2e-3


@pytest.mark.parametrize("kernel", ["auto", "simt"])
def test_tiny_config_through_the_oracle_pipeline(cuda_ok, kernel):
    """The tiny configuration end to end from the oracle's own case (joint
    SVD, factors, latent rows): whichever split kernel the dims select."""
    from oracle import inputs as oi
    from tests.gpu_util import GpuCase
    case = oi.build_case(synthetic.CONFIGS[0])
    kern = {"auto": q.QSVD_KERNEL_AUTO, "simt": q.QSVD_KERNEL_SIMT}[kernel]
    got, ws = GpuCase(case, kernel=kern).decode()
    assert int(ws[:4].view(torch.int32).item()) == 0
    assert rel_err(got, case.reference()) <= 1e-4
