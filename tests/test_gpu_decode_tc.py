"""Parity of the tensor-core split kernels (tcgen05 + TMA, absorbed query,
fp16/bf16 latent, int4/int8 latent with group scales) against the fp64
oracle and against the CUDA-core kernel.  The 16-bit cases run both
tensor-core variants: one CTA per split (CTA) and the tile's channels spread
over a thread-block cluster (CL; r = 256 -> 2 CTAs, 384 -> 3, 768 -> 3,
1536 -> 6, 2048 -> 8).

Bar: max |o_gpu - o_ref| / rms(o_ref) <= 2e-3 (P and the absorbed query are
rounded to the latent's 16-bit type before the MMA; accumulation is fp32).
"""
import numpy as np
import pytest
import torch

import rank_joint_qkv_b200 as q
import synthetic
from oracle import inputs as oi
from tests.gpu_util import GpuCase, rel_err

pytestmark = pytest.mark.gpu
TOL = 2e-3
TC = q.QSVD_KERNEL_TCGEN05
CTA, CL = q.QSVD_KERNEL_TCGEN05_CTA, q.QSVD_KERNEL_TCGEN05_CLUSTER
BOTH = [CTA, CL]


def kernel_ran(ws):
    """Split kernel recorded in the workspace header."""
    return int(ws[12:16].view(torch.int32).item())

_CASES = {}


def case(key):
    if key not in _CASES:
        base = synthetic.SHRUNK[1]   # E=512, H=4, r=256, B=3, L=300 (ragged tail)
        w = {
            "f16": base,
            "bf16": synthetic.replace(base, cache="bf16", weight="bf16"),
            "h32": synthetic.replace(base, E=4096, H=32, r=384, B=2, L=520),
            "r768": synthetic.replace(base, E=1024, H=8, r=768, B=2, L=700),
            "full": synthetic.replace(base, B=2, L=512),       # whole tiles only
            # quantised latents: per-group S buffers, dequantised Z
            "i4": synthetic.SHRUNK[3],                           # r 384, H2, ragged tail
            "i8": synthetic.replace(synthetic.SHRUNK[3], cache="i8", name="shrunk-int8-h2"),
            "i4h32": synthetic.replace(synthetic.SHRUNK[3], E=4096, H=32, r=768, B=2, L=600,
                                       h2_n=256),
            # r 256: two channel groups, four Z items per tile
            "i4r256": synthetic.replace(synthetic.SHRUNK[3], r=256, h2_n=0, h2_m=0),
            "i8r256": synthetic.replace(synthetic.SHRUNK[3], r=256, h2_n=0, h2_m=0, cache="i8",
                                        name="shrunk-int8-r256"),
            "i4r256rag": synthetic.replace(synthetic.SHRUNK[3], r=256, h2_n=0, h2_m=0, B=4, L=700,
                                           ragged=(1, 700)),
            # r 1536 at 32 heads: twelve Z chunks leave TMEM for one S group buffer
            "i8r1536": synthetic.replace(synthetic.SHRUNK[3], E=4096, H=32, r=1536, B=2, L=300,
                                         h2_n=0, h2_m=0, cache="i8", name="shrunk-int8-r1536"),
            "i4r1536": synthetic.replace(synthetic.SHRUNK[3], E=4096, H=32, r=1536, B=2, L=300,
                                         h2_n=0, h2_m=0, name="shrunk-int4-r1536"),
            # cluster shapes: 6 CTAs of 256 channels (the LLaVA-7B rank), 8 of 256
            "c6": synthetic.replace(base, E=4096, H=32, r=1536, B=2, L=300),
            "c6bf": synthetic.replace(base, E=4096, H=32, r=1536, B=2, L=290, cache="bf16",
                                      weight="bf16"),
            "c8": synthetic.replace(base, E=2048, H=16, r=2048, B=2, L=280),
        }[key]
        _CASES[key] = _build(w)
    return _CASES[key]


def _build(w):
    if w.E > 1024:
        # direct seeded factors: skips the E x 3E SVD, which decode parity does not need
        wuq, wuk, wuv = (a.astype(np.float64) for a in synthetic.direct_up_weights_np(w))
        wd = synthetic.direct_down_weight_np(w).astype(np.float64)
        return oi.build_case(w, factors_override=(0.5, (wd, wuq, wuk, wuv), None))
    return oi.build_case(w)


_KEYS16 = ["full", "f16", "bf16", "h32", "r768", "c6", "c6bf", "c8"]


@pytest.mark.parametrize("key,kern", [(k, v) for k in _KEYS16 for v in BOTH] +
                         [(k, CTA) for k in ("i4", "i8", "i4h32", "i4r256", "i8r256", "i4r256rag",
                                             "i8r1536", "i4r1536")])
def test_tc_matches_oracle(cuda_ok, key, kern):
    c = case(key)
    g = GpuCase(c, kernel=kern)
    got, ws = g.decode()
    assert q.status_word(ws) == 0
    assert kernel_ran(ws) == kern
    err = rel_err(got, c.reference())
    assert err <= TOL, f"{key}: {err:.3e}"


@pytest.mark.parametrize("key,kern", [("f16", CTA), ("f16", CL), ("bf16", CTA), ("bf16", CL),
                                      ("c6", CL), ("i4", CTA), ("i8", CTA)])
def test_tc_agrees_with_simt(cuda_ok, key, kern):
    c = case(key)
    a, _ = GpuCase(c, kernel=kern).decode()
    b, _ = GpuCase(c, kernel=q.QSVD_KERNEL_SIMT).decode()
    assert rel_err(a, b) <= TOL


def test_tc_auto_picks_one_cta_per_split(cuda_ok):
    """The default and the generic tensor-core request run one CTA per split
    (faster than the cluster kernel on the 16-bit workloads measured); the
    cluster kernel runs when asked for."""
    for kern in (q.QSVD_KERNEL_AUTO, TC):
        for key in ("f16", "i4"):
            _, ws = GpuCase(case(key), kernel=kern).decode()
            assert kernel_ran(ws) == CTA
    _, ws = GpuCase(case("f16"), kernel=CL).decode()
    assert kernel_ran(ws) == CL


@pytest.mark.parametrize("kern", BOTH)
@pytest.mark.parametrize("splits", [1, 2, 3, 7, 1000])
def test_tc_split_invariance(cuda_ok, splits, kern):
    c = case("h32")
    g = GpuCase(c, kernel=kern)
    base, _ = g.decode(num_splits=1)
    got, ws = g.decode(num_splits=splits)
    assert q.status_word(ws) == 0
    # each split rounds P = 2^(s - m_split) to fp16 against its own reference
    # max, so split counts differ at the level of fp16 rounding (2^-11)
    assert rel_err(got, base) <= 1e-3
    assert rel_err(got, c.reference()) <= TOL


@pytest.mark.parametrize("key", ["i4", "i8r256"])
@pytest.mark.parametrize("splits", [1, 3, 1000])
def test_tc_int_split_invariance(cuda_ok, key, splits):
    """Quantised latents at any split count (each converting warp's share of
    items changes with the split boundaries)."""
    c = case(key)
    got, ws = GpuCase(c, kernel=CTA).decode(num_splits=splits)
    assert q.status_word(ws) == 0
    assert rel_err(got, c.reference()) <= TOL


@pytest.mark.parametrize("kern", BOTH)
@pytest.mark.parametrize("lens", [[1, 0, 2], [127, 128, 129], [255, 256, 257], [300, 1, 300]])
def test_tc_edge_lengths(cuda_ok, lens, kern):
    w = synthetic.replace(synthetic.SHRUNK[1], B=len(lens), ragged=None, L=max(lens))
    c = oi.build_case(w, lengths=np.array(lens, np.int32))
    got, ws = GpuCase(c, kernel=kern).decode(num_splits=2)
    for b, n in enumerate(lens):
        if n == 0:
            assert np.all(got[b] == 0.0)
    assert rel_err(got, c.reference()) <= TOL
    assert q.status_word(ws) == 0


@pytest.mark.parametrize("kern", BOTH)
def test_tc_nan_padding_rows(cuda_ok, kern):
    """NaN in rows past each length (ragged tiles are zero-filled on load)."""
    c = case("f16")
    g = GpuCase(c, kernel=kern)
    for b, n in enumerate(c.lengths):
        g.cache[b, int(n):] = float("nan")
    got, _ = g.decode(num_splits=4)
    assert np.all(np.isfinite(got))
    assert rel_err(got, c.reference()) <= TOL


@pytest.mark.parametrize("kern", BOTH)
def test_tc_large_score_range_rescales(cuda_ok, kern):
    """Scores spanning far more than 2^8 between tiles force the conditional
    rescale of the latent accumulator."""
    c = case("full")
    g = GpuCase(c, kernel=kern)
    # grow the latent along the sequence: later tiles dominate the softmax
    caches, lens = [], c.lengths
    w = c.w
    for b in range(w.B):
        n = int(lens[b])
        ramp = np.linspace(0.2, 3.0, n)[:, None]
        vals = c.caches[b] * ramp
        dev = oi.to_device_dtype(vals, w.cache)
        g.cache[b, :n] = oi.as_torch(dev, w.cache).to("cuda")
        caches.append(oi.from_device_dtype(dev, w.cache))
    c2 = oi.Case(**{**c.__dict__, "caches": caches})
    got, ws = g.decode(num_splits=1)
    assert q.status_word(ws) == 0
    assert rel_err(got, c2.reference()) <= TOL


# Rotary mode: keys rebuilt on the tensor cores (K_h = C W^u_{k,h}, two heads
# per MMA), rotated and scored by CUDA cores; then the softmax and latent
# accumulation on the given scores -- on the tensor cores when r % 128 == 0
# and H <= 32 (Z only, two MMA issuers on alternating 128-channel chunks),
# else on CUDA cores (r = 320 below).
_ROPE = {}


def rope_case(key):
    if key not in _ROPE:
        base = synthetic.SHRUNK[2]
        w = {"s2": base,                                     # bf16, r 256, even H
             "s4": synthetic.SHRUNK[4],                      # bf16, r 384 (odd chunk count), H 5, ragged
             "s2f16": synthetic.replace(base, cache="f16", weight="f16"),
             "h32": synthetic.replace(base, E=4096, H=32, r=384, B=2, L=520),
             # heads padded to 48; Z of all chunks beyond TMEM: two CTAs per
             # split, 9 + 9 chunks (r 2304) and 6 + 5 chunks (r 1408)
             "h40": synthetic.replace(synthetic.SHRUNK[4], E=5120, H=40, r=2304, B=2, L=300,
                                      ragged=(150, 300)),
             "h40r1408": synthetic.replace(base, E=5120, H=40, r=1408, B=2, L=280),
             "h40r384": synthetic.replace(base, E=5120, H=40, r=384, B=2, L=260),
             "h32r2304": synthetic.replace(base, E=4096, H=32, r=2304, B=2, L=270),
             "r320": synthetic.replace(base, r=320)}[key]    # CUDA-core softmax on given scores
        _ROPE[key] = _build(w)
    return _ROPE[key]


@pytest.mark.parametrize("key", ["s2", "s4", "s2f16", "h32", "h40", "h40r1408", "h40r384",
                                 "h32r2304", "r320"])
def test_tc_rope_matches_oracle(cuda_ok, key):
    c = rope_case(key)
    got, ws = GpuCase(c, kernel=TC).decode()
    assert q.status_word(ws) == 0
    err = rel_err(got, c.reference())
    assert err <= TOL, f"{key}: {err:.3e}"


@pytest.mark.parametrize("key", ["s2", "s4", "h32", "h40"])
def test_tc_rope_agrees_with_simt(cuda_ok, key):
    c = rope_case(key)
    a, _ = GpuCase(c, kernel=TC).decode()
    b, _ = GpuCase(c, kernel=q.QSVD_KERNEL_SIMT).decode()
    assert rel_err(a, b) <= TOL


@pytest.mark.parametrize("key,splits", [("h32", 1), ("h32", 3), ("h32", 1000), ("h40", 1),
                                        ("h40", 7)])
def test_tc_rope_split_invariance(cuda_ok, key, splits):
    c = rope_case(key)
    got, ws = GpuCase(c, kernel=TC).decode(num_splits=splits)
    assert q.status_word(ws) == 0
    assert rel_err(got, c.reference()) <= TOL


@pytest.mark.parametrize("lens", [[1, 0, 2], [127, 128, 129], [300, 1, 257]])
def test_tc_rope_edge_lengths(cuda_ok, lens):
    w = synthetic.replace(synthetic.SHRUNK[2], B=len(lens), ragged=None, L=max(lens))
    c = oi.build_case(w, lengths=np.array(lens, np.int32))
    got, ws = GpuCase(c, kernel=TC).decode(num_splits=2)
    for b, n in enumerate(lens):
        if n == 0:
            assert np.all(got[b] == 0.0)
    assert rel_err(got, c.reference()) <= TOL
    assert q.status_word(ws) == 0


def test_tc_rope_nan_padding_rows(cuda_ok):
    """NaN in rows past each length: neither the keys nor the latent
    accumulation of the given-scores pass may pick them up."""
    c = rope_case("s4")
    g = GpuCase(c, kernel=TC)
    for b, n in enumerate(c.lengths):
        g.cache[b, int(n):] = float("nan")
    got, _ = g.decode(num_splits=4)
    assert np.all(np.isfinite(got))
    assert rel_err(got, c.reference()) <= TOL


@pytest.mark.parametrize("key", ["s4", "r320"])
def test_tc_rope_split_passes_as_separate_calls(cuda_ok, key):
    """The rotary split run as its two passes (scores, then the softmax and
    latent accumulation), each its own call, gives the one-call result."""
    c = rope_case(key)
    g = GpuCase(c, kernel=TC)
    whole, _ = g.decode(num_splits=5)
    parts, ws = g.decode(num_splits=5, phases_separately=True,
                         split_phases=(q.QSVD_PHASE_SPLIT_SCORES, q.QSVD_PHASE_SPLIT_ACCUM))
    assert q.status_word(ws) == 0
    assert np.array_equal(whole, parts)
