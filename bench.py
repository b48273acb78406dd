"""Benchmark of one decode step of joint-QKV latent attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 1]
                    [--impl ours|reference] [--splits G] [--kernel auto|simt|tcgen05]

One step = the whole hot path for one batch: append the current token of
every sequence (c = x W^d, written as row len-1), then decode attention over
the latent cache (query projection and absorption, split-KV flash decoding,
cross-split merge and value up-projection).  Inputs are synthetic and seeded
(``synthetic``); the latent cache is far larger than L2.  The timed region
is exactly K steps of a CUDA-graph replay, repeated back to back until about
0.3 s have passed (so the clock record holds enough samples) and reported as
the median region; a second figure times single steps after a 256 MB write
that flushes L2.  At N = 1 the line also carries the other workloads (int4
and int8 latents, the two rotary layers), each with its own roofline.
Prints one JSON line (rank 0).

Multi-GPU (torchrun): every rank holds its own batch of sequences (weak
scaling, no collective on the data path); the step time is the max over
ranks.  ``--impl reference`` times the CPU oracle on this host's cores on a
bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time
from typing import Optional

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synthetic  # noqa: E402

METRIC = "decode-attn KV-tokens/s over C_qkv latent cache; achieved HBM GB/s vs peak"
UNIT = "KV-tokens/s"
TORCH_DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
CALIB_SEQS, CALIB_LEN = 256, 640   # calibration set: sequences x tokens (image + text)
ROW_BYTES = {"f32": 4, "f16": 2, "bf16": 2, "i8": 1, "i4": 0.5}


# ---------------------------------------------------------------------------
# inputs
# ---------------------------------------------------------------------------

def workload(cfg: int, cache: Optional[str] = None):
    """Configuration ``cfg``; ``cache`` overrides its latent type (the int4
    workload also runs with an int8 latent: same shapes, 780 bytes a token)."""
    w = synthetic.CONFIGS[cfg]
    if cache and cache != w.cache:
        w = synthetic.replace(w, cache=cache, name=w.name.replace(w.cache.replace("i", "int"),
                                                                  cache.replace("i", "int")))
    return w


def bench_inputs(cfg: int, device: str, rank: int = 0, cache: Optional[str] = None):
    """Device-resident synthetic inputs of configuration ``cfg`` (the same
    recipe on every rank, seeded by rank)."""
    w = workload(cfg, cache)
    lens = synthetic.lengths(w)
    max_len = int(lens.max())
    cs, _ = synthetic.direct_channel_scales(w)
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed * 7919 + rank)
    B, r = w.B, w.r
    cs_t = torch.tensor(cs, dtype=torch.float32, device=device)
    scales = None
    if w.cache in ("f32", "f16", "bf16"):
        cache = torch.empty((B, max_len, r), dtype=TORCH_DT[w.cache], device=device)
        for b in range(B):   # per sequence keeps the fp32 temporary small
            rows = torch.randn((max_len, r), generator=gen, device=device) * cs_t
            cache[b].copy_(rows)
    else:
        # rows drawn as in the 16-bit case, then quantised per (token, group):
        # fp16 scale = group amax / qmax, code = rint(value / scale) (the
        # latent quantiser's own rule), int4 packed two codes per byte
        g, qmax = w.group, (7 if w.cache == "i4" else 127)
        cache = torch.empty((B, max_len, r if w.cache == "i8" else r // 2),
                            dtype=torch.int8 if w.cache == "i8" else torch.uint8, device=device)
        scales = torch.empty((B, max_len, r // g), dtype=torch.float16, device=device)
        for b in range(B):
            rows = (torch.randn((max_len, r), generator=gen, device=device) * cs_t).view(max_len, r // g, g)
            sc = (rows.abs().amax(dim=2) / qmax).to(torch.float16)
            codes = torch.round(rows / sc.float().clamp_min(1e-30)[..., None]).clamp_(-qmax, qmax)
            codes = codes.to(torch.int8).view(max_len, r)
            scales[b].copy_(sc)
            if w.cache == "i8":
                cache[b].copy_(codes)
            else:
                cache[b].copy_(((codes[:, 0::2] & 0xF) | ((codes[:, 1::2] & 0xF) << 4)).to(torch.uint8))
    wuq, wuk, wuv = (torch.from_numpy(a).to(device=device, dtype=TORCH_DT[w.weight])
                     for a in synthetic.direct_up_weights_np(w))
    wd = torch.from_numpy(synthetic.direct_down_weight_np(w)).to(device=device,
                                                               dtype=TORCH_DT[w.weight])
    x = torch.from_numpy(synthetic.direct_new_tokens_np(w)).to(dtype=TORCH_DT[w.weight])
    return dict(w=w, lens=lens, max_len=max_len, cache=cache, scales=scales, wuq=wuq, wuk=wuk,
                wuv=wuv, wd=wd, x_host=x)


def latent_bytes(w, lens) -> float:
    """Latent-cache bytes one step reads: rows x row bytes (+ group scales)."""
    rows = float(np.sum(lens))
    b = rows * w.r * ROW_BYTES[w.cache]
    if w.cache in ("i8", "i4"):
        b += rows * (w.r // w.group) * 2
    return b


def weight_bytes(w) -> float:
    """W^d and the three W^u read once per step (4 r E elements)."""
    return 4.0 * w.r * w.E * (4 if w.weight == "f32" else 2)


# ---------------------------------------------------------------------------
# clocks, peaks, profiles
# ---------------------------------------------------------------------------

class ClockSampler:
    """SM clock and clock-event reasons sampled while the timed region runs:
    NVML from a thread every 5 ms (the timed region can be tens of ms),
    else nvidia-smi every 100 ms.  Reads only; changes no GPU setting."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.thread = None
        self.lines = []

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(self.gpu)
        bus = "%08x:%02x:%02x.0" % (getattr(props, "pci_domain_id", 0), props.pci_bus_id,
                                    props.pci_device_id)
        return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())

    def _nvml_loop(self, nv, h):
        names = [("hw_slowdown", nv.nvmlClocksEventReasonHwSlowdown),
                 ("hw_thermal_slowdown", nv.nvmlClocksEventReasonHwThermalSlowdown),
                 ("sw_thermal_slowdown", nv.nvmlClocksEventReasonSwThermalSlowdown),
                 ("sw_power_cap", nv.nvmlClocksEventReasonSwPowerCap)]
        mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        while not self.stop.is_set():
            sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
            rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
            flags = ["Active" if rs & bit else "Not Active" for _, bit in names]
            self.lines.append(",".join([str(self.gpu), str(sm), str(mx), "0", hex(rs)] + flags))
            time.sleep(0.005)

    def __enter__(self):
        import threading
        try:
            nv, h = self._nvml_handle()
            self.stop = threading.Event()
            self.thread = threading.Thread(target=self._nvml_loop, args=(nv, h), daemon=True)
            self.thread.start()
            return self
        except Exception:
            self.thread = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=2)
            return
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            p = [x.strip() for x in l.split(",")]
            if len(p) < 9:
                continue
            try:
                sm.append(float(p[1]))
                mx = float(p[2])
            except ValueError:
                continue
            for n, v in zip(names, p[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def measured_peaks():
    """HBM copy GB/s, bf16 TFLOP/s burst and sustained, and whose numbers."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return (float(d["hbm_gbs"]), float(d["bf16_tflops"]),
                float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured")
    return 6650.0, 1590.0, 1400.0, "fallback"


def kernel_source_hash(files) -> str:
    """Hash of the code in the kernel's source files, comments and whitespace
    left out: a committed DRAM-traffic figure stays valid across comment
    edits and goes stale with any change of code."""
    import re
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "rank_joint_qkv_b200", "csrc", f)) as fh:
            src = fh.read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
        src = re.sub(r"//[^\n]*", " ", src)
        h.update(" ".join(src.split()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(kernel_name: str, workload: str, src_files):
    """DRAM bytes per launch of the split kernel from the committed ncu
    summary, if it was taken on the current kernel source; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel_name, {}).get(workload)
    if not e or e.get("source_sha") != kernel_source_hash(src_files):
        return None
    return float(e["dram_bytes_per_launch"])


def agreed_regions(run_region, min_ms: float, world: int, device):
    """run_region() (-> ms) back to back until min_ms have passed (at least
    once).  With several ranks the decision is taken together after every
    region (a MAX all-reduce of "wants more"), so every rank runs the same
    number of regions and the barriers inside them stay paired."""
    regions, spent = [], 0.0
    while True:
        regions.append(float(run_region()))
        spent += regions[-1]
        more = spent < min_ms
        if world > 1:
            t = torch.tensor([1.0 if more else 0.0], device=device)
            torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
            more = t.item() > 0.0
        if not more:
            return regions


def max_over_ranks(x: float, device, world: int) -> float:
    """Max of a per-rank scalar over the process group (no-op for one rank)."""
    if world <= 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_step_per_rank: float, steps: int, world: int, ms_max: float) -> float:
    """Whole-job throughput: every rank's units over the slowest rank's time."""
    return units_per_step_per_rank * steps * world / (ms_max / 1e3)


# ---------------------------------------------------------------------------
# our implementation
# ---------------------------------------------------------------------------

class DecodeStep:
    """One decode step of a workload on this rank's GPU: append the current
    token of every sequence, then the decode phases, each one API call.
    Rotary mode on the tensor cores runs the split as its two passes so that
    the scores pass (the dominant kernel there) is timed on its own."""

    def __init__(self, q, cfg, cache_override, args, device, rank):
        self.q = q
        inp = bench_inputs(cfg, device, rank, cache=cache_override)
        self.inp = inp
        w, lens, max_len = inp["w"], inp["lens"], inp["max_len"]
        self.w, self.lens, self.max_len, self.device = w, lens, max_len, device
        kern = {"auto": q.QSVD_KERNEL_AUTO, "simt": q.QSVD_KERNEL_SIMT,
                "tcgen05": q.QSVD_KERNEL_TCGEN05, "cta": q.QSVD_KERNEL_TCGEN05_CTA,
                "cluster": q.QSVD_KERNEL_TCGEN05_CLUSTER}[args.kernel]
        self.splits = args.splits
        self.dims = q.make_dims(w.E, w.H, w.d_h, w.r, w.B, max_len, cache=w.cache, weight=w.weight,
                                out="f32", group=w.group, rope=w.rope, rope_base=w.rope_base,
                                kernel=kern, out_proj=args.out_proj)
        self.packed = q.qsvd_prepare_weights(self.dims, inp["wd"], inp["wuq"], inp["wuk"], inp["wuv"])
        if args.out_proj != "none":
            # synthetic output projection W_O (E x E), seeded like the other weights
            gwo = torch.Generator(device=device).manual_seed(w.seed * 31 + 5)
            wo = (torch.randn((w.E, w.E), generator=gwo, device=device) / math.sqrt(w.E)).to(TORCH_DT[w.weight])
            q.qsvd_prepare_out_proj(self.dims, wo, self.packed)
            del wo
        self.stream = torch.cuda.current_stream()
        self.lens_dev = torch.from_numpy(lens).to(device)
        self.pos_dev = (self.lens_dev - 1).to(torch.int32)
        self.x_dev = inp["x_host"].to(device)
        self.cnew = torch.empty((w.B, w.r), dtype=torch.float32, device=device)
        self.out = torch.empty((w.B, w.E), dtype=torch.float32, device=device)
        self.app_ws = torch.empty(q.append_workspace_bytes(self.dims), dtype=torch.uint8, device=device)
        self.dec_ws = torch.empty(q.decode_workspace_bytes(self.dims, self.splits), dtype=torch.uint8,
                                  device=device)
        # which split kernel these dims run (workspace header), from one full call
        self._append(self.stream)
        self._decode(q.QSVD_PHASE_ALL, self.stream)
        torch.cuda.synchronize()
        self.kernel_used = int(self.dec_ws[12:16].view(torch.int32).item())
        self.rope_tc = w.rope and self.kernel_used == q.QSVD_KERNEL_TCGEN05_CTA
        split_phases = ([("scores", q.QSVD_PHASE_SPLIT_SCORES), ("accum", q.QSVD_PHASE_SPLIT_ACCUM)]
                        if self.rope_tc else [("split", q.QSVD_PHASE_SPLIT)])
        self.phases = ([("append", None), ("prologue", q.QSVD_PHASE_PROLOGUE)] + split_phases +
                       [("combine", q.QSVD_PHASE_COMBINE)])
        self.graph = None

    def _append(self, st):
        self.q.qsvd_append_latent(self.dims, self.packed, self.x_dev, self.pos_dev, self.inp["cache"],
                                  self.inp["scales"], self.cnew, None, self.app_ws, stream=st)

    def _decode(self, ph, st):
        self.q.qsvd_decode_attn(self.dims, self.packed, self.cnew, True, self.inp["cache"],
                                self.inp["scales"], self.lens_dev, self.out, num_splits=self.splits,
                                workspace=self.dec_ws, phases=ph, stream=st)

    def step(self, ev=None, st=None):
        """ev: len(phases) + 1 events bracketing the phases."""
        st = self.stream if st is None else st
        for k, (name, ph) in enumerate(self.phases):
            if ev is not None:
                ev[k].record(st)
            if ph is None:
                self._append(st)
            else:
                self._decode(ph, st)
        if ev is not None:
            ev[len(self.phases)].record(st)

    def eager_pass(self, steps):
        """The API calls per step with events between the phases: per-phase
        mean times, the dominant kernel's per-launch times, kernels per step."""
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(self.phases) + 1)]
              for _ in range(steps)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n0 = self.q.kernel_launches()
        torch.cuda.synchronize()
        t0.record(self.stream)
        for i in range(steps):
            self.step(ev[i])
        t1.record(self.stream)
        torch.cuda.synchronize()
        per_step = (self.q.kernel_launches() - n0) // steps
        phase_ms = {name: statistics.mean(e[k].elapsed_time(e[k + 1]) for e in ev)
                    for k, (name, _) in enumerate(self.phases)}
        dom = 2   # the split (absorbed) or the scores pass (rotary)
        dom_ms = [e[dom].elapsed_time(e[dom + 1]) for e in ev]
        return t0.elapsed_time(t1), phase_ms, dom_ms, per_step

    def capture(self):
        """One step captured as a CUDA graph: the same kernels with the same
        arguments, without the host work between launches."""
        gstream = torch.cuda.Stream(self.device)
        gstream.wait_stream(self.stream)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph, stream=gstream):
            self.step(st=gstream)
        for _ in range(3):
            self.graph.replay()
        torch.cuda.synchronize()

    def run(self):
        if self.graph is not None:
            self.graph.replay()
        else:
            self.step()

    def timed_regions(self, steps, world, min_seconds):
        """Regions of exactly `steps` steps, each bracketed by a barrier and a
        synchronize, repeated back to back until `min_seconds` have passed
        (at least one; every rank runs the same number): per-region ms."""
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

        def region():
            torch.cuda.synchronize()
            if world > 1:
                torch.distributed.barrier()
            t0.record(self.stream)
            for _ in range(steps):
                self.run()
            t1.record(self.stream)
            torch.cuda.synchronize()
            if world > 1:
                torch.distributed.barrier()
            return t0.elapsed_time(t1)

        return agreed_regions(region, min_seconds * 1e3, world, self.device)

    def flushed_steps(self, n, flush):
        """n steps, each preceded by a write of `flush` (a buffer larger than
        L2) and timed alone: per-step milliseconds."""
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(n)]
        torch.cuda.synchronize()
        for a, b in ev:
            flush.fill_(1)
            a.record(self.stream)
            self.run()
            b.record(self.stream)
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in ev]

    def roofline(self, dom_ms):
        """Roofline object of the dominant kernel from its per-launch times."""
        q, w = self.q, self.w
        hbm_peak, tc_burst, tc_sustained, peak_kind = measured_peaks()
        dom_mean = statistics.mean(dom_ms)
        lat_b = latent_bytes(w, self.lens)
        kname = ("k_rope_scores" if self.rope_tc
                 else "k_split_cl" if self.kernel_used == q.QSVD_KERNEL_TCGEN05_CLUSTER
                 else "k_split_tc" if self.kernel_used == q.QSVD_KERNEL_TCGEN05_CTA
                 else "k_split_rope" if w.rope else "k_split_abs")
        src = (["split_cluster.cu", "tc_common.cuh", "internal.cuh"] if kname == "k_split_cl"
               else ["split_tc.cu", "tc_common.cuh", "internal.cuh"] if kname in ("k_split_tc", "k_rope_scores")
               else ["split_simt.cu", "internal.cuh"])
        traffic = profiled_traffic(kname, w.name, src)
        if self.rope_tc:
            # keys rebuilt per head: K_h = C W^u_{k,h}, 2 r E flop per valid token
            flops = 2.0 * w.r * w.E * float(np.sum(self.lens))
            achieved = flops / (dom_mean / 1e3) / 1e12
            # the scores kernel runs back to back inside long runs of steps (the
            # power cap sets its clock): the sustained GEMM peak is its ceiling
            return {"bound": "tensor", "achieved": achieved, "peak": tc_sustained, "unit": "TFLOP/s",
                    "frac": achieved / tc_sustained, "traffic": traffic, "kernel": kname,
                    "peak_kind": peak_kind + " bf16 sustained (fp16 has the same dense rate)",
                    "frac_of_burst_peak": achieved / tc_burst,
                    "flops_per_launch": flops, "launch_ms": dom_mean,
                    "launch_ms_median": statistics.median(dom_ms)}
        achieved = lat_b / (dom_mean / 1e3) / 1e9
        return {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                "frac": achieved / hbm_peak, "traffic": traffic,
                "kernel": kname, "peak_kind": peak_kind,
                "bytes_per_launch": lat_b, "launch_ms": dom_mean,
                "launch_ms_median": statistics.median(dom_ms)}


def other_workloads(q, args, device):
    """The other workloads of the path, each timed in this run on its own
    inputs: its dominant kernel's roofline and its graph-replayed step.
    Parity cases of the test suite, reported here so that one bench line
    carries every workload's measured fraction."""
    out = []
    for cfg, cache in ((3, None), (3, "i8"), (2, None), (4, None)):
        st = DecodeStep(q, cfg, cache, args, device, 0)
        for _ in range(3):
            st.step()
        _, phase_ms, dom_ms, _ = st.eager_pass(args.extra_steps)
        st.capture()
        regions = st.timed_regions(args.extra_steps, 1, 0.0)
        ms = regions[0] / args.extra_steps
        tokens = float(np.sum(st.lens))
        out.append({"workload": st.w.name, "cache": st.w.cache,
                    "mode": "rope" if st.w.rope else "absorbed",
                    "tokens_per_step": int(tokens), "ms_per_step": ms,
                    "value": tokens / (ms / 1e3), "unit": UNIT,
                    "step_hbm_gbs": (latent_bytes(st.w, st.lens) + weight_bytes(st.w)) / (ms / 1e3) / 1e9,
                    "phase_ms": phase_ms, "roofline": st.roofline(dom_ms),
                    "steps": args.extra_steps})
        del st
        torch.cuda.empty_cache()
    return out


def run_ours(args, rank, world, local_rank):
    import rank_joint_qkv_b200 as q

    device = f"cuda:{local_rank}"
    torch.cuda.set_device(device)
    st = DecodeStep(q, args.config, args.cache, args, device, rank)
    w, lens, max_len = st.w, st.lens, st.max_len
    for _ in range(args.warmup):
        st.step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()

    ms_eager, phase_ms, dom_ms, launches_per_step = st.eager_pass(args.steps)
    ms_eager = max_over_ranks(ms_eager, device, world)
    if not args.eager:
        st.capture()
    # the timed region: exactly K steps, repeated back to back until about
    # 0.3 s have passed so that the clock record holds enough samples; the
    # reported time is the median region's
    with ClockSampler(torch.cuda.current_device()) as clk:
        regions = st.timed_regions(args.steps, world, args.min_region_s)
    ms = statistics.median(regions)
    ms_max = max_over_ranks(ms, device, world)
    launches = launches_per_step * args.steps
    tokens_per_step = float(np.sum(lens))
    value = whole_job_rate(tokens_per_step, args.steps, world, ms_max)

    # L2 flushed before every step (a 256 MB write), each step timed alone
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    fl = st.flushed_steps(max(10, min(args.steps, 50)), flush)
    del flush
    fl_ms = max_over_ranks(statistics.median(fl), device, world)

    # end to end through the public API with host buffers
    x_pin = st.inp["x_host"].pin_memory()
    lens_pin = torch.from_numpy(lens).pin_memory()
    out_pin = torch.empty((w.B, w.E), dtype=torch.float32).pin_memory()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ke = max(3, args.steps)
    torch.cuda.synchronize()
    e0.record(st.stream)
    for _ in range(ke):
        st.x_dev.copy_(x_pin, non_blocking=True)
        st.lens_dev.copy_(lens_pin, non_blocking=True)
        torch.sub(st.lens_dev, 1, out=st.pos_dev)
        st.step()
        out_pin.copy_(st.out, non_blocking=True)
    e1.record(st.stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), device, world)
    e2e_value = whole_job_rate(tokens_per_step, ke, world, e2e_ms)
    h2d = x_pin.numel() * x_pin.element_size() + lens_pin.numel() * 4
    d2h = out_pin.numel() * 4

    if rank != 0:
        return None
    lat_b = latent_bytes(w, lens)
    step_gbs = (lat_b + weight_bytes(w)) / (ms_max / args.steps / 1e3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.cache, "data": "synthetic",
        "config": {"workload": w.name, "E": w.E, "H": w.H, "d_h": w.d_h, "r": w.r,
                   "batch_per_gpu": w.B, "kv_len": int(max_len),
                   "tokens_per_step_per_gpu": int(tokens_per_step), "cache": w.cache,
                   "weights": w.weight, "mode": "rope" if w.rope else "absorbed",
                   "splits": args.splits, "kernel": args.kernel, "out_proj": args.out_proj,
                   "l2": "inputs larger than L2: %.0f MB latent read per step per GPU; "
                         "l2_flushed: the same step after a 256 MB write, timed alone"
                         % (lat_b / 1e6),
                   "parallelism": f"dp{world}"},
        "steps_per_s": args.steps * 1e3 / ms_max,
        "timing": ("CUDA-graph replay of one captured step (the kernels of the four API calls)"
                   if st.graph is not None else "eager API calls"),
        "timed_regions": {"count": len(regions), "steps_each": args.steps,
                          "ms_median": statistics.median(regions), "ms_min": min(regions),
                          "ms_max": max(regions)},
        "ms_per_step_eager": ms_eager / args.steps,
        "phase_ms": phase_ms,
        "step_hbm_gbs": step_gbs,
        "l2_flushed": {"ms_per_step": fl_ms, "value": whole_job_rate(tokens_per_step, 1, world, fl_ms),
                       "steps": len(fl), "stat": "median"},
        "roofline": st.roofline(dom_ms),
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h)},
        "gpu_launches": int(launches),
        "gpu_launches_all_regions": int(launches * len(regions)),
    }
    line["clocks"] = clk.summary()
    del st
    torch.cuda.empty_cache()
    if world == 1 and not args.no_extra and args.config == 1 and args.cache is None:
        line["other_workloads"] = other_workloads(q, args, device)
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, lens, budget_s=args.cpu_seconds)
    return line


# ---------------------------------------------------------------------------
# CPU oracle (baseline leg and reference arm)
# ---------------------------------------------------------------------------

def oracle_sample(w, n_tokens: int, b: int):
    """One sequence of the workload on the host: latent rows, new latent, W^u."""
    from oracle import qsvd_ref as ref   # noqa: F401  (checked import for the timed leg)
    c = synthetic.direct_latent_rows_np(w, b, n_tokens).astype(np.float64)
    cnew = synthetic.direct_new_latent_np(w)[b:b + 1].astype(np.float64)
    wuq, wuk, wuv = (a.astype(np.float64) for a in synthetic.direct_up_weights_np(w))
    return c, cnew, wuq, wuk, wuv


def time_oracle(w, n_tokens, budget_s, max_seqs=None):
    """The oracle on sequences of n_tokens: until budget_s seconds are spent,
    or exactly max_seqs sequences when that is given."""
    from oracle import qsvd_ref as ref
    rb = w.rope_base if w.rope else None
    done_tokens, spent, seqs = 0, 0.0, 0
    while (seqs < max_seqs) if max_seqs is not None else (spent < budget_s):
        c, cnew, wuq, wuk, wuv = oracle_sample(w, n_tokens, seqs % w.B)
        t = time.perf_counter()
        ref.decode_materialized([c], [n_tokens], cnew, wuq, wuk, wuv, w.H, rope_base=rb)
        spent += time.perf_counter() - t
        done_tokens += n_tokens
        seqs += 1
    return done_tokens, spent, seqs


def cpu_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_baseline(w, lens, budget_s=15.0):
    n = int(min(int(np.max(lens)), 8192))
    tokens, spent, seqs = time_oracle(w, n, budget_s)
    return {"value": tokens / spent, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
            "sample": f"{seqs} sequence(s) of {n} tokens through the fp64 oracle "
                      f"(keys/values materialised), {spent:.1f} s"}


def run_prefill(args):
    """qsvd_prefill_latent on the workload's whole cache (every token of every
    sequence, B x L rows): one GEMM x W^d with the cache's rounding or
    quantisation fused, timed with CUDA events over K launches."""
    import rank_joint_qkv_b200 as q
    device = "cuda:0"
    torch.cuda.set_device(device)
    w = synthetic.CONFIGS[args.config]
    max_len = w.L
    n = w.B * max_len
    dims = q.make_dims(w.E, w.H, w.d_h, w.r, w.B, max_len, cache=w.cache, weight=w.weight,
                       group=w.group)
    wt = torch.bfloat16 if w.weight == "bf16" else torch.float16
    g = torch.Generator(device=device).manual_seed(w.seed)
    wd = (torch.randn(w.E, w.r, device=device, generator=g) / math.sqrt(w.E)).to(wt)
    wu = torch.zeros(w.r, w.E, dtype=wt, device=device)
    packed = q.qsvd_prepare_weights(dims, wd, wu, wu, wu)
    x = torch.randn(n, w.E, device=device, generator=g).to(wt)
    rowb = {"f16": 2 * w.r, "bf16": 2 * w.r, "f32": 4 * w.r, "i8": w.r, "i4": w.r // 2}[w.cache]
    cache = torch.empty(n, rowb, dtype=torch.uint8, device=device)
    scales = (torch.empty(n, w.r // w.group, dtype=torch.float16, device=device)
              if w.cache in ("i4", "i8") else None)
    dst = torch.arange(n, dtype=torch.int32, device=device)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    for _ in range(args.warmup):
        q.qsvd_prefill_latent(dims, packed, x, dst, cache, scales, None, status)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        e0.record()
        for _ in range(args.steps):
            q.qsvd_prefill_latent(dims, packed, x, dst, cache, scales, None, status)
        e1.record()
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    flops = 2.0 * n * w.E * w.r
    achieved = flops / (ms / 1e3) / 1e12
    _, burst, sustained, kind = measured_peaks()
    return {"metric": "prefill latent rows/s (x W^d, rounded or quantised into the cache)",
            "value": n / (ms / 1e3), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "dtype": w.weight, "data": "synthetic",
            "config": {"workload": w.name, "E": w.E, "r": w.r, "rows": n, "cache": w.cache},
            "roofline": {"bound": "tensor", "achieved": achieved, "unit": "TFLOP/s",
                         "peak": sustained, "frac": achieved / sustained,
                         "frac_of_burst_peak": achieved / burst, "peak_kind": kind + " bf16 sustained",
                         "kernel": "k_prefill", "flops_per_launch": flops},
            "status": int(status.item()), "clocks": clk.summary()}


def run_prefill_attn(args):
    """qsvd_prefill_attention over every prompt of the workload (B prompts of
    L tokens: Q, K, V rebuilt from the latent rows by three GEMMs, then causal
    attention on the tensor cores), timed with CUDA events over K calls."""
    import rank_joint_qkv_b200 as q
    device = "cuda:0"
    torch.cuda.set_device(device)
    w = synthetic.CONFIGS[args.config]
    inp = bench_inputs(args.config, device)
    lens = inp["lens"]
    max_len = inp["max_len"]
    dims = q.make_dims(w.E, w.H, w.d_h, w.r, w.B, max_len, cache=w.cache, weight=w.weight,
                       rope=w.rope, rope_base=w.rope_base)
    packed = q.qsvd_prepare_weights(dims, inp["wd"], inp["wuq"], inp["wuk"], inp["wuv"])
    lens_dev = torch.from_numpy(lens).to(device)
    out = torch.empty((w.B, max_len, w.E), dtype=torch.float32, device=device)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    ws = torch.empty(q.prefill_attention_workspace_bytes(dims), dtype=torch.uint8, device=device)
    for _ in range(args.warmup):
        q.qsvd_prefill_attention(dims, packed, inp["cache"], lens_dev, out, status, workspace=ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n0 = q.kernel_launches()
    with ClockSampler(torch.cuda.current_device()) as clk:
        e0.record()
        for _ in range(args.steps):
            q.qsvd_prefill_attention(dims, packed, inp["cache"], lens_dev, out, status, workspace=ws)
        e1.record()
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    L = lens.astype(np.float64)
    rows = float(w.B * max_len)
    attn_flops = float(np.sum(2.0 * w.E * L * (L + 1.0)))      # causal Q K^T and P V
    gemm_flops = 3 * 2.0 * rows * w.r * w.E                      # Q, K, V = C W^u
    flops = attn_flops + gemm_flops
    achieved = flops / (ms / 1e3) / 1e12
    _, burst, sustained, kind = measured_peaks()
    parts = 3.0   # S: 3 part products; P V: 3 part products
    return {"metric": "prefill attention prompt tokens/s (Q, K, V rebuilt from the latent rows, causal)",
            "value": float(np.sum(L)) / (ms / 1e3), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "dtype": w.cache,
            "data": "synthetic",
            "config": {"workload": w.name + "-prefill-attention", "E": w.E, "H": w.H, "r": w.r,
                       "prompts": w.B, "prompt_len": int(max_len), "rope": bool(w.rope)},
            "roofline": {"bound": "tensor", "achieved": achieved, "unit": "TFLOP/s", "peak": sustained,
                         "frac": achieved / sustained, "frac_of_burst_peak": achieved / burst,
                         "peak_kind": kind + " bf16 sustained", "traffic": None,
                         "kernel": "qsvd_prefill_attention (3 latent GEMMs, 3 part kernels, k_prefill_attn)",
                         "flops_per_call": flops, "attention_flops": attn_flops, "gemm_flops": gemm_flops,
                         "tensor_work_per_attention_flop": parts},
            "gpu_launches": q.kernel_launches() - n0, "status": int(status.item()),
            "clocks": clk.summary()}


def run_beta(args):
    """One split-exponent evaluation of the calibration objective per step
    (factors for beta, layout with H2, three prefills, two decodes, the
    squared output error on the host) on the workload's shapes with
    ``CALIB_SEQS`` synthetic calibration sequences of ``CALIB_LEN`` tokens;
    the oracle's objective timed beside it on a bounded sample of them."""
    import rank_joint_qkv_b200 as q
    from rank_joint_qkv_b200.calibrate import BetaObjective
    device = "cuda:0"
    torch.cuda.set_device(device)
    w = synthetic.CONFIGS[args.config]
    n_seq, L = CALIB_SEQS, CALIB_LEN
    g = torch.Generator(device=device).manual_seed(w.seed * 131 + 7)
    # leading singular triplets of a joint [W_Q W_K W_V]: orthonormal columns / rows
    u = torch.linalg.qr(torch.randn(w.E, w.r, generator=g, device=device))[0]
    vt = torch.linalg.qr(torch.randn(3 * w.E, w.r, generator=g, device=device))[0].T.contiguous()
    sig = synthetic.spectrum(w.E)[: w.r]
    x = torch.randn(n_seq * L, w.E, generator=g, device=device)
    x[:, torch.from_numpy(synthetic.outlier_channels(w)).to(device)] *= w.outlier_scale
    x = x.to(TORCH_DT[w.weight])
    lens = np.full(n_seq, L, np.int64)
    h2_m = w.h2_m if w.h2_n else 0
    h2_q = synthetic.small_orthogonal(h2_m) if h2_m else None
    obj = BetaObjective(u, sig, vt, x, lens, w.H, cache=w.cache, group=w.group, weight=w.weight,
                        h2_q=h2_q, h2_m=h2_m)
    betas = [0.5 + 0.4 * math.sin(1.7 * k) for k in range(args.warmup + args.steps)]
    for b in betas[: args.warmup]:
        obj(b)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    vals = [obj(b) for b in betas[args.warmup:]]
    dt = (time.perf_counter() - t0) / args.steps
    flops = 2 * 2.0 * n_seq * L * w.E * w.r     # the two full prefills dominate
    line = {"metric": "beta-search objective evaluations/s (calibration latents quantised, decode-step outputs)",
            "value": 1.0 / dt, "unit": "evaluations/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "dtype": w.weight, "data": "synthetic",
            "config": {"workload": w.name, "E": w.E, "H": w.H, "r": w.r, "cache": w.cache,
                       "h2": f"H_{w.r // h2_m} x Q_{h2_m} folded" if h2_m else None,
                       "calibration": f"{n_seq} sequences x {L} tokens"},
            "timing": "host wall clock per evaluation, including the two B x E outputs read back",
            "prefill_flop_per_step": flops, "objective_sample": vals[:3],
            "status": obj.status_word()}
    # the oracle on a bounded sample: the same objective for a few sequences
    from oracle import beta_ref as br
    k = 2
    u64, vt64 = u.double().cpu().numpy(), vt.double().cpu().numpy()
    s_full = np.asarray(sig, np.float64)
    xs = [x[i * L:(i + 1) * L].float().cpu().numpy().astype(np.float64) for i in range(k)]
    h2 = None
    if h2_m:
        from oracle import qsvd_ref as ref
        h2 = ref.h2_matrix(w.r // h2_m, h2_q)
    t0 = time.perf_counter()
    br.calibration_objective(u64, s_full, vt64, w.r, 0.5, xs, lens[:k], w.H,
                             bits=4 if w.cache == "i4" else 8, group=w.group, weight=w.weight, h2=h2)
    cdt = (time.perf_counter() - t0) * n_seq / k
    line["cpu_baseline"] = {"value": 1.0 / cdt, "unit": "evaluations/s", "cores": torch.get_num_threads(),
                            "kind": "oracle",
                            "sample": f"{k} of {n_seq} calibration sequences, scaled by {n_seq // k}"}
    return line


def run_per_head(args):
    """qsvd_decode_attn_per_head on the workload's shapes with per-head key
    and value latents of rank ``--per-head-rank``: K launches timed with
    CUDA events; HBM figure = latent bytes per launch / launch time."""
    import rank_joint_qkv_b200 as q
    device = "cuda:0"
    torch.cuda.set_device(device)
    w = synthetic.CONFIGS[args.config]
    r = args.per_head_rank
    cache = w.cache if w.cache in ("f16", "bf16", "f32") else "f16"
    wt = TORCH_DT[w.weight]
    g = torch.Generator(device=device).manual_seed(w.seed * 17 + 3)
    lat = torch.empty((w.B, w.H, w.L, r), dtype=TORCH_DT[cache], device=device)
    lat_v = torch.empty_like(lat)
    for t in (lat, lat_v):
        for b in range(w.B):   # per sequence keeps the fp32 temporary small
            t[b].copy_(torch.randn((w.H, w.L, r), generator=g, device=device))
    bk = (torch.randn((w.H, r, w.d_h), generator=g, device=device) / math.sqrt(r)).to(wt)
    bv = (torch.randn((w.H, r, w.d_h), generator=g, device=device) / math.sqrt(r)).to(wt)
    qv = torch.randn((w.B, w.E), generator=g, device=device)
    lens = torch.full((w.B,), w.L, dtype=torch.int32, device=device)
    dims = q.make_dims(w.E, w.H, w.d_h, r, w.B, w.L, cache=cache, weight=w.weight, rope=w.rope,
                       rope_base=w.rope_base)
    out = torch.empty((w.B, w.E), dtype=torch.float32, device=device)
    ws = torch.empty(q.per_head_workspace_bytes(dims), dtype=torch.uint8, device=device)
    for _ in range(args.warmup):
        q.qsvd_decode_attn_per_head(dims, bk, bv, qv, lat, lat_v, lens, out, workspace=ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n0 = q.kernel_launches()
    with ClockSampler(torch.cuda.current_device()) as clk:
        e0.record()
        for _ in range(args.steps):
            q.qsvd_decode_attn_per_head(dims, bk, bv, qv, lat, lat_v, lens, out, workspace=ws)
        e1.record()
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    lat_b = 2.0 * lat.numel() * lat.element_size()
    hbm, _, _, kind = measured_peaks()
    gbs = lat_b / (ms / 1e3) / 1e9
    return {"metric": "per-head latent decode KV-tokens/s (key and value latents per head)",
            "value": w.B * w.L / (ms / 1e3), "unit": "KV-tokens/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "dtype": cache,
            "data": "synthetic",
            "config": {"workload": w.name + "-per-head", "E": w.E, "H": w.H, "d_h": w.d_h, "r_per_head": r,
                       "mode": "rope" if w.rope else "absorbed",
                       "batch": w.B, "kv_len": w.L, "cache": cache, "weights": w.weight},
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                         "traffic": None, "kernel": "qsvd_decode_attn_per_head (all its kernels)",
                         "peak_kind": kind, "bytes_per_launch": lat_b},
            "gpu_launches": q.kernel_launches() - n0, "clocks": clk.summary()}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    w = workload(args.config, args.cache)
    lens = synthetic.lengths(w)
    n = int(min(int(np.max(lens)), 8192))
    for _ in range(args.warmup):
        time_oracle(w, min(n, 512), 0.0, max_seqs=1)
    # one sequence per step; its length bounded so that the K steps take
    # about two minutes at most (the oracle's cost grows with the tokens)
    t1, s1, _ = time_oracle(w, min(n, 1024), 0.0, max_seqs=1)
    per_token = s1 / t1
    n = int(max(128, min(n, 120.0 / (max(1, args.steps) * per_token))))
    tokens, spent, seqs = 0, 0.0, 0
    for _ in range(args.steps):
        t, s, k = time_oracle(w, n, 0.0, max_seqs=1)
        tokens += t
        spent += s
        seqs += k
    value = tokens / spent
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": spent / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.name, "E": w.E, "H": w.H, "d_h": w.d_h, "r": w.r,
                   "mode": "rope" if w.rope else "absorbed",
                   "sample_per_step": f"one sequence of {n} tokens"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
                         "sample": f"{seqs} sequence(s) of {n} tokens, one per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=int, default=1)
    ap.add_argument("--cache", choices=["i4", "i8"], default=None,
                    help="latent type of a quantised workload (the int4 workload also runs with int8)")
    ap.add_argument("--min-region-s", type=float, default=0.3,
                    help="repeat the K-step timed region until this many seconds have passed")
    ap.add_argument("--extra-steps", type=int, default=30,
                    help="steps per timed region of the other workloads")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the other workloads' measurements")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--splits", type=int, default=0)
    ap.add_argument("--kernel", choices=["auto", "simt", "tcgen05", "cta", "cluster"], default="auto")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--out-proj", choices=["none", "chain", "fold"], default="none",
                    help="apply the layer's output projection W_O in the combine (chain: V-up then "
                         "W_O; fold: W^u_v folded into W_O per head)")
    ap.add_argument("--per-head-rank", type=int, default=0,
                    help="time the per-head latent decode (key and value latents of this rank per head)")
    ap.add_argument("--beta-search", action="store_true",
                    help="time one evaluation of the split-exponent calibration objective per step")
    ap.add_argument("--prefill", action="store_true",
                    help="time qsvd_prefill_latent over the workload's whole cache instead of a decode step")
    ap.add_argument("--prefill-attn", action="store_true",
                    help="time qsvd_prefill_attention over the workload's prompts (all B x L tokens)")
    ap.add_argument("--eager", action="store_true",
                    help="time the API calls as issued instead of a CUDA-graph replay of one step")
    ap.add_argument("--batch", type=int, default=0,
                    help="prefill-attention and per-head modes only: this many sequences instead of "
                         "the workload's own B (a smaller case, e.g. for a profiler capture)")
    args = ap.parse_args()
    if args.batch:
        if not (args.prefill_attn or args.per_head_rank):
            ap.error("--batch applies to --prefill-attn and --per-head-rank only")
        synthetic.CONFIGS[args.config] = synthetic.replace(synthetic.CONFIGS[args.config], B=args.batch)
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.prefill:
        line = run_prefill(args)
    elif args.prefill_attn:
        line = run_prefill_attn(args)
    elif args.beta_search:
        line = run_beta(args)
    elif args.per_head_rank:
        line = run_per_head(args)
    elif args.impl == "reference":
        line = run_reference(args, rank, world)
    else:
        if world > 1:
            import datetime
            torch.cuda.set_device(local_rank)
            torch.distributed.init_process_group(
                "nccl", timeout=datetime.timedelta(seconds=300),
                device_id=torch.device(f"cuda:{local_rank}"))
        try:
            line = run_ours(args, rank, world, local_rank)
        finally:
            if world > 1:
                torch.distributed.destroy_process_group()
    if rank == 0 and line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
