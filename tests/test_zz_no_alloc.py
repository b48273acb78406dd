"""The allocation-free append (qsvd_append_latent_static) against the
workspace entry point (qsvd_append_latent).

The static variant exists for callers that cannot allocate device memory --
an engine or plugin host that only passes the call's own tensors, or a
deployment whose memory budget is fixed after start-up -- so it keeps its
split-K scratch in a library-owned static device array instead of a
workspace.  Both entry points run the same kernels, so the stored cache
bytes, the fp16 scales and the fp32 latent must agree bit for bit; two calls
in a row with different tokens check that the shared scratch carries nothing
over from one call to the next.

This file sorts last so that a run stopping at the first failure has run
every other test; it also passes alone in a fresh process (the first call on
a device performs the static array's address lookup).
"""
import ctypes

import numpy as np
import pytest
import torch

import rank_joint_qkv_b200 as q
from oracle import inputs as oi


def _setup(E, r, B, cache_dtype, max_len, seed):
    g = np.random.default_rng(seed)
    dims = q.make_dims(E, E // 128, 128, r, B, max_len, cache=cache_dtype, weight="f16")
    dev = "cuda"
    f16 = lambda a: oi.as_torch(oi.to_device_dtype(a, "f16"), "f16").to(dev)
    wd = f16(g.standard_normal((E, r)) / np.sqrt(E))
    wu = f16(g.standard_normal((r, E)) / np.sqrt(r))
    packed = q.qsvd_prepare_weights(dims, wd, wu, wu, wu)
    rowb = {"f16": 2 * r, "i8": r, "i4": r // 2}[cache_dtype]

    def buffers():
        cache = torch.zeros((B, max_len, rowb), dtype=torch.uint8, device=dev)
        scales = (torch.zeros((B, max_len, r // 128), dtype=torch.float16, device=dev)
                  if cache_dtype in ("i8", "i4") else None)
        c_out = torch.zeros((B, r), dtype=torch.float32, device=dev)
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        return cache, scales, c_out, status

    tokens = [f16(g.standard_normal((B, E))) for _ in range(2)]
    pos = [torch.from_numpy((np.arange(B) * (k + 3)) % max_len).to(dev, torch.int32)
           for k in range(2)]
    return dims, packed, buffers, tokens, pos


@pytest.mark.gpu
@pytest.mark.parametrize("cache_dtype", ["i4", "f16"])
def test_static_append_matches_workspace_append(cuda_ok, cache_dtype):
    E, r, B, max_len = 4096, 768, 32, 64
    dims, packed, buffers, tokens, pos = _setup(E, r, B, cache_dtype, max_len, 11)
    ref_bufs, got_bufs = buffers(), buffers()
    lib = ctypes.CDLL(q.LIB_PATH)
    lib.qsvd_append_latent_static.argtypes = q._sigs["qsvd_append_latent_static"]
    lib.qsvd_append_latent_static.restype = ctypes.c_int
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for k in range(2):   # two calls in a row through the shared scratch
        cache, scales, c_out, status = ref_bufs
        q.qsvd_append_latent(dims, packed, tokens[k], pos[k], cache, scales, c_out, status)
        cache, scales, c_out, status = got_bufs
        st = lib.qsvd_append_latent_static(
            ctypes.byref(dims), ctypes.c_void_p(packed.data_ptr()),
            ctypes.c_void_p(tokens[k].data_ptr()), ctypes.c_void_p(pos[k].data_ptr()),
            ctypes.c_void_p(cache.data_ptr()),
            None if scales is None else ctypes.c_void_p(scales.data_ptr()),
            ctypes.c_void_p(c_out.data_ptr()), ctypes.c_void_p(status.data_ptr()), stream)
        assert st == q.QSVD_OK
        torch.cuda.synchronize()
        for a, b in zip(ref_bufs, got_bufs):
            if a is not None:
                assert torch.equal(a, b), f"call {k}"
    assert int(got_bufs[3].item()) == 0


def test_static_append_rejects_oversize_requests():
    """batch 512, r 4096: even ksplit = 1 needs 2,097,152 floats > 1,048,576."""
    dims = q.make_dims(4096, 32, 128, 4096, 512, 16, cache="f16", weight="f16")
    lib = ctypes.CDLL(q.LIB_PATH)
    lib.qsvd_append_latent_static.argtypes = q._sigs["qsvd_append_latent_static"]
    lib.qsvd_append_latent_static.restype = ctypes.c_int
    p = ctypes.c_void_p(1 << 20)   # never dereferenced: the size check fails first
    st = lib.qsvd_append_latent_static(ctypes.byref(dims), p, p, p, p, None, None, None, None)
    assert st == q.QSVD_ERR_WORKSPACE
    assert b"static scratch" in q._lib.qsvd_last_error()


def test_static_append_rejects_misaligned_pointers():
    """x and cache are read and written with vector accesses, so, as with the
    workspace entry point, a pointer off a 16-byte boundary is refused on the
    host before anything is enqueued (the pointers are never dereferenced)."""
    dims = q.make_dims(1024, 8, 128, 256, 4, 16, cache="f16", weight="f16")
    lib = ctypes.CDLL(q.LIB_PATH)
    lib.qsvd_append_latent_static.argtypes = q._sigs["qsvd_append_latent_static"]
    lib.qsvd_append_latent_static.restype = ctypes.c_int
    good = ctypes.c_void_p(1 << 20)
    bad = ctypes.c_void_p((1 << 20) + 2)
    for x, cache in ((bad, good), (good, bad)):
        st = lib.qsvd_append_latent_static(ctypes.byref(dims), good, x, good, cache, None, None,
                                           None, None)
        assert st == q.QSVD_ERR_INVALID_ARG
        assert b"16-byte aligned" in q._lib.qsvd_last_error()
    odd = ctypes.c_void_p((1 << 20) + 1)   # fp16 scales are stored two bytes at a time
    d8 = q.make_dims(1024, 8, 128, 256, 4, 16, cache="i8", weight="f16")
    st = lib.qsvd_append_latent_static(ctypes.byref(d8), good, good, good, good, odd, None, None, None)
    assert st == q.QSVD_ERR_INVALID_ARG
    assert b"scales must be 2-byte" in q._lib.qsvd_last_error()
