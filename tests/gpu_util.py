"""Helpers that move an oracle test case onto the GPU and run it through the
C-ABI (via the thin binding).  The inputs are the oracle's own arrays; the
library never sees anything the oracle did not also consume."""
import numpy as np
import torch

import rank_joint_qkv_b200 as q
from oracle import inputs as oi

DEV = "cuda"


def rel_err(got: np.ndarray, ref: np.ndarray) -> float:
    """max |got - ref| / rms(ref) over the whole output."""
    ref = np.asarray(ref, np.float64)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    return float(np.max(np.abs(np.asarray(got, np.float64) - ref))) / max(rms, 1e-30)


def dims_for(case, *, kernel=q.QSVD_KERNEL_SIMT, out="f32", h2=False, h2_m=0, max_len=None):
    w = case.w
    return q.make_dims(w.E, w.H, w.d_h, w.r, w.B, case.max_len if max_len is None else max_len,
                       cache=w.cache, weight=w.weight, out=out, group=w.group, rope=w.rope,
                       rope_base=w.rope_base, kernel=kernel, h2=h2, h2_m=h2_m)


def dev_tensor(a: np.ndarray, dtype: str) -> torch.Tensor:
    return oi.as_torch(a, dtype).to(DEV)


class GpuCase:
    """Device copies of a Case plus a prepared weight buffer."""

    def __init__(self, case, *, kernel=q.QSVD_KERNEL_SIMT, out="f32"):
        self.case = case
        w = case.w
        self.dims = dims_for(case, kernel=kernel, out=out)
        self.wd = dev_tensor(case.wd_dev, w.weight)
        self.wuq = dev_tensor(case.wuq_dev, w.weight)
        self.wuk = dev_tensor(case.wuk_dev, w.weight)
        self.wuv = dev_tensor(case.wuv_dev, w.weight)
        self.packed = q.qsvd_prepare_weights(self.dims, self.wd, self.wuq, self.wuk, self.wuv)
        cd = w.cache if w.cache in ("f32", "f16", "bf16") else ("i8" if w.cache == "i8" else "i4")
        self.cache = dev_tensor(case.cache_dev, cd)
        self.scales = (torch.from_numpy(case.scales_dev).to(DEV)
                       if case.scales_dev is not None else None)
        self.lengths = torch.from_numpy(np.asarray(case.lengths, np.int32)).to(DEV)
        self.cnew = torch.from_numpy(case.cnew).to(DEV)
        self.out_dtype = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[out]

    def decode(self, *, num_splits=0, lengths=None, phases_separately=False, qin=None,
               qin_is_latent=True, split_phases=None):
        w = self.case.w
        out = torch.full((w.B, w.E), float("nan"), dtype=self.out_dtype, device=DEV)
        lens = self.lengths if lengths is None else lengths
        qi = self.cnew if qin is None else qin
        if not phases_separately:
            ws = q.qsvd_decode_attn(self.dims, self.packed, qi, qin_is_latent, self.cache,
                                    self.scales, lens, out, num_splits=num_splits)
        else:
            ws = None
            for ph in (q.QSVD_PHASE_PROLOGUE,) + tuple(split_phases or (q.QSVD_PHASE_SPLIT,)):
                ws = q.qsvd_decode_attn(self.dims, self.packed, qi, qin_is_latent, self.cache,
                                        self.scales, lens, out, num_splits=num_splits,
                                        workspace=ws, phases=ph)
            q.qsvd_combine_splits(self.dims, self.packed, ws, num_splits, lens, out)
        torch.cuda.synchronize()
        return out.float().cpu().numpy(), ws
