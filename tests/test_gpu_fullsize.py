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


# cfg 1: fp16 absorbed (tensor cores); cfg 3: int4 + H2 workload (tensor
# cores, quantised latent); cfg 2 / 4: bf16 rotary (CUDA cores).  cfg 4's
# oracle samples its two shortest sequences (keys and values of a
# 32k-token sequence are 1.3 GB each in float64).
@pytest.mark.parametrize("cfg,kernel", [(1, "auto"), (3, "auto"), (2, "auto"), (4, "auto")])
def test_fullsize_sampled(cuda_ok, cfg, kernel):
    dev = "cuda"
    inp = bench.bench_inputs(cfg, dev)
    w, lens, max_len = inp["w"], inp["lens"], inp["max_len"]
    kern = {"auto": q.QSVD_KERNEL_AUTO, "simt": q.QSVD_KERNEL_SIMT,
            "tcgen05": q.QSVD_KERNEL_TCGEN05}[kernel]
    dims = q.make_dims(w.E, w.H, w.d_h, w.r, w.B, max_len, cache=w.cache, weight=w.weight,
                       group=w.group, rope=w.rope, rope_base=w.rope_base, kernel=kern)
    packed = q.qsvd_prepare_weights(dims, inp["wd"], inp["wuq"], inp["wuk"], inp["wuv"])
    cnew = synthetic.direct_new_latent_np(w)
    out = torch.empty((w.B, w.E), dtype=torch.float32, device=dev)
    lens_dev = torch.from_numpy(lens).to(dev)
    q.qsvd_decode_attn(dims, packed, torch.from_numpy(cnew).to(dev), True, inp["cache"],
                       inp["scales"], lens_dev, out)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    wuq, wuk, wuv = (t.float().cpu().numpy().astype(np.float64)
                     for t in (inp["wuq"], inp["wuk"], inp["wuv"]))
    rb = w.rope_base if w.rope else None
    picks = (0, w.B - 1) if cfg != 4 else tuple(int(i) for i in np.argsort(lens)[:2])
    for b in picks:
        n = int(lens[b])
        c = _latent_rows(inp, w, b, n)
        want = ref.decode_materialized([c], [n], cnew[b:b + 1].astype(np.float64), wuq, wuk,
                                       wuv, w.H, rope_base=rb)
        assert rel_err(got[b:b + 1], want) <= 2e-3
