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
from tests.gpu_util import rel_err

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("cfg,kernel", [(1, "auto")])
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
    for b in (0, w.B - 1):
        n = int(lens[b])
        c = inp["cache"][b, :n].float().cpu().numpy().astype(np.float64)
        want = ref.decode_materialized([c], [n], cnew[b:b + 1].astype(np.float64), wuq, wuk,
                                       wuv, w.H, rope_base=rb)
        assert rel_err(got[b:b + 1], want) <= 2e-3
