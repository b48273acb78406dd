"""Python binding of the joint-QKV latent decode library (libqsvd.so, sm_100a).

Argument marshalling only: every step of the decode path runs in the CUDA
kernels of ``libqsvd.so``; PyTorch supplies device memory and streams.  The
functions carry the C names of ``include/qsvd.h`` and raise ``QsvdError`` on a
non-OK status.  Importing the package fails loudly when the library has not
been built (``python rank_joint_qkv_b200/build.py``): there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqsvd.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python rank_joint_qkv_b200/build.py`")

_lib = ctypes.CDLL(LIB_PATH)

# ----------------------------------------------------------------- constants
QSVD_OK, QSVD_ERR_INVALID_ARG, QSVD_ERR_UNSUPPORTED, QSVD_ERR_WORKSPACE, QSVD_ERR_CUDA = range(5)
QSVD_F32, QSVD_F16, QSVD_BF16, QSVD_I8, QSVD_I4 = range(5)
QSVD_TILE_TOKENS = 128
QSVD_PHASE_PROLOGUE, QSVD_PHASE_SPLIT, QSVD_PHASE_COMBINE, QSVD_PHASE_ALL = 1, 2, 4, 7
QSVD_PHASE_SPLIT_SCORES, QSVD_PHASE_SPLIT_ACCUM = 8, 16
QSVD_STATUS_LEN_CLAMPED, QSVD_STATUS_POS_OOB, QSVD_STATUS_SCALE_SAT, QSVD_STATUS_TIMEOUT = 1, 2, 4, 8
QSVD_KERNEL_AUTO, QSVD_KERNEL_SIMT, QSVD_KERNEL_TCGEN05 = 0, 1, 2
QSVD_KERNEL_TCGEN05_CTA, QSVD_KERNEL_TCGEN05_CLUSTER = 3, 4
QSVD_OUT_PROJ_NONE, QSVD_OUT_PROJ_CHAIN, QSVD_OUT_PROJ_FOLD = 0, 1, 2
QSVD_PER_HEAD_HEAD_MAJOR, QSVD_PER_HEAD_TOKEN_MAJOR = 0, 1
OUT_PROJ_CODE = {None: QSVD_OUT_PROJ_NONE, "none": QSVD_OUT_PROJ_NONE,
                 "chain": QSVD_OUT_PROJ_CHAIN, "fold": QSVD_OUT_PROJ_FOLD}

DTYPE_CODE = {"f32": QSVD_F32, "f16": QSVD_F16, "bf16": QSVD_BF16, "i8": QSVD_I8, "i4": QSVD_I4}


class qsvd_dims(ctypes.Structure):
    _fields_ = [
        ("E", ctypes.c_int), ("H", ctypes.c_int), ("d_h", ctypes.c_int), ("r", ctypes.c_int),
        ("batch", ctypes.c_int), ("max_len", ctypes.c_int), ("group", ctypes.c_int),
        ("rope", ctypes.c_int), ("rope_base", ctypes.c_float),
        ("softmax_scale", ctypes.c_float), ("cache_dtype", ctypes.c_int),
        ("weight_dtype", ctypes.c_int), ("out_dtype", ctypes.c_int), ("h2", ctypes.c_int),
        ("h2_m", ctypes.c_int), ("kernel", ctypes.c_int), ("out_proj", ctypes.c_int),
    ]


_P = ctypes.c_void_p
_SZ = ctypes.POINTER(ctypes.c_size_t)
_D = ctypes.POINTER(qsvd_dims)
_sigs = {
    "qsvd_prepare_weights": [_D, _P, _P, _P, _P, _P, _P, _SZ, _P],
    "qsvd_append_latent": [_D, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P],
    "qsvd_decode_attn": [_D, _P, _P, ctypes.c_int, _P, _P, _P, ctypes.c_int, _P, _SZ, _P,
                         ctypes.c_uint, _P],
    "qsvd_combine_splits": [_D, _P, _P, ctypes.c_int, _P, _P, _P],
    "qsvd_append_latent_static": [_D, _P, _P, _P, _P, _P, _P, _P, _P],
    "qsvd_prefill_latent": [_D, _P, _P, ctypes.c_int, _P, _P, _P, _P, _P, _P],
    "qsvd_prepare_out_proj": [_D, _P, _P, ctypes.c_size_t, _P],
    "qsvd_split_factors": [_D, _P, _P, _P, _P, _P, _P, _P, _P, _P],
    "qsvd_decode_attn_per_head": [_D, _P, _P, _P, _P, _P, _P, ctypes.c_int, _P, _SZ, _P, _P],
    "qsvd_testing_set_score_wait_ns": [ctypes.c_ulonglong],
    "qsvd_prefill_attention": [_D, _P, _P, _P, _P, _SZ, _P, _P, _P],
    "qsvd_prepare_per_head_fold": [_D, _P, _P, _P, _P],
    "qsvd_beta_exponents": [_P, ctypes.c_int, ctypes.c_double, _P, _P, _P],
    "qsvd_sq_diff_sum": [_P, _P, ctypes.c_int64, _P, _P],
}
for _name, _args in _sigs.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = ctypes.c_int
_lib.qsvd_status_string.argtypes = [ctypes.c_int]
_lib.qsvd_status_string.restype = ctypes.c_char_p
_lib.qsvd_last_error.argtypes = []
_lib.qsvd_last_error.restype = ctypes.c_char_p
_lib.qsvd_kernel_launches.argtypes = []
_lib.qsvd_kernel_launches.restype = ctypes.c_uint64
_lib.qsvd_abi_version.argtypes = []
_lib.qsvd_abi_version.restype = ctypes.c_int


class QsvdError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.qsvd_last_error().decode(errors="replace")
        name = _lib.qsvd_status_string(status).decode()
        super().__init__(f"{where}: {name}: {msg}")


def _check(status: int, where: str):
    if status != QSVD_OK:
        raise QsvdError(status, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def make_dims(E, H, d_h, r, batch, max_len, *, cache="f16", weight="f16", out="f32",
              group=128, rope=False, rope_base=10000.0, softmax_scale=0.0, h2=False,
              h2_m=0, kernel=QSVD_KERNEL_AUTO, out_proj=None) -> qsvd_dims:
    """``out_proj``: None/"none", "chain" or "fold" (see QSVD_OUT_PROJ_*)."""
    return qsvd_dims(E, H, d_h, r, batch, max_len, group, int(bool(rope)), float(rope_base),
                     float(softmax_scale), DTYPE_CODE[cache], DTYPE_CODE[weight],
                     DTYPE_CODE[out], int(bool(h2)), int(h2_m), int(kernel),
                     OUT_PROJ_CODE[out_proj])


def kernel_launches() -> int:
    return int(_lib.qsvd_kernel_launches())


def abi_version() -> int:
    return int(_lib.qsvd_abi_version())


def qsvd_testing_set_score_wait_ns(ns: int) -> None:
    """Failure-detection tests only: with ns != 0 the tensor-core split
    kernel's softmax warps wait on a barrier nothing releases, giving up
    after ns nanoseconds (current device); 0 turns it off."""
    _check(_lib.qsvd_testing_set_score_wait_ns(int(ns)), "qsvd_testing_set_score_wait_ns")


def _empty_bytes(n: int, device) -> torch.Tensor:
    return torch.empty(max(int(n), 256), dtype=torch.uint8, device=device)


def qsvd_prepare_weights(dims: qsvd_dims, wd, wuq, wuk, wuv, h2_q=None, packed=None,
                         stream=None) -> torch.Tensor:
    """Lay out W^d, W^u_q, W^u_k, W^u_v (device tensors) into a packed buffer.
    ``h2_q``: optional (m x m) float32 CPU array/tensor, the small factor of
    H2 = H_{r/m} (x) Q.  Returns the packed device buffer."""
    n = ctypes.c_size_t(0)
    _check(_lib.qsvd_prepare_weights(ctypes.byref(dims), None, None, None, None, None, None,
                                     ctypes.byref(n), None), "qsvd_prepare_weights(size)")
    if packed is None:
        packed = _empty_bytes(n.value, wd.device)
    n = ctypes.c_size_t(packed.numel() * packed.element_size())
    hq = None
    if h2_q is not None:
        hq = torch.as_tensor(h2_q, dtype=torch.float32).contiguous().cpu()
    _check(_lib.qsvd_prepare_weights(ctypes.byref(dims), _ptr(wd), _ptr(wuq), _ptr(wuk),
                                     _ptr(wuv), _ptr(hq), _ptr(packed), ctypes.byref(n),
                                     _stream(stream)), "qsvd_prepare_weights")
    return packed


def qsvd_prepare_out_proj(dims: qsvd_dims, wo, packed, stream=None):
    """Add W_O (E x E device tensor, y = o W_O) to a buffer filled by
    qsvd_prepare_weights with the same dims (dims.out_proj chain or fold)."""
    _check(_lib.qsvd_prepare_out_proj(ctypes.byref(dims), _ptr(wo), _ptr(packed),
                                      packed.numel() * packed.element_size(), _stream(stream)),
           "qsvd_prepare_out_proj")


def qsvd_split_factors(dims: qsvd_dims, u, vt, a, b, wd, wuq, wuk, wuv, stream=None):
    """Fill wd (E x r) and wuq/wuk/wuv (r x E), weight-dtype device tensors,
    with U diag(a) and diag(b) V^T (u: E x r, vt: r x 3E, a, b: r; float32
    device tensors)."""
    _check(_lib.qsvd_split_factors(ctypes.byref(dims), _ptr(u), _ptr(vt), _ptr(a), _ptr(b), _ptr(wd),
                                   _ptr(wuq), _ptr(wuk), _ptr(wuv), _stream(stream)),
           "qsvd_split_factors")


def append_workspace_bytes(dims: qsvd_dims) -> int:
    n = ctypes.c_size_t(0)
    _check(_lib.qsvd_append_latent(ctypes.byref(dims), None, None, None, None, None, None,
                                   None, None, ctypes.byref(n), None),
           "qsvd_append_latent(size)")
    return n.value


def qsvd_append_latent(dims: qsvd_dims, packed, x, pos, cache, scales=None, c_out=None,
                       status=None, workspace=None, stream=None):
    if workspace is None:
        workspace = _empty_bytes(append_workspace_bytes(dims), x.device)
    n = ctypes.c_size_t(workspace.numel() * workspace.element_size())
    _check(_lib.qsvd_append_latent(ctypes.byref(dims), _ptr(packed), _ptr(x), _ptr(pos),
                                   _ptr(cache), _ptr(scales), _ptr(c_out), _ptr(status),
                                   _ptr(workspace), ctypes.byref(n), _stream(stream)),
           "qsvd_append_latent")
    return workspace


def qsvd_prefill_latent(dims: qsvd_dims, packed, x, dst_rows, cache, scales=None,
                        c_out=None, status=None, stream=None):
    """Latent rows of x.shape[0] tokens at once, row i stored at cache row
    dst_rows[i] (b * max_len + t)."""
    _check(_lib.qsvd_prefill_latent(ctypes.byref(dims), _ptr(packed), _ptr(x), int(x.shape[0]),
                                    _ptr(dst_rows), _ptr(cache), _ptr(scales), _ptr(c_out),
                                    _ptr(status), _stream(stream)),
           "qsvd_prefill_latent")


def qsvd_beta_exponents(sigma, beta: float, a, b, stream=None) -> None:
    """a = sigma^beta, b = sigma^(1 - beta) (float64 powers), device tensors."""
    _check(_lib.qsvd_beta_exponents(_ptr(sigma), int(sigma.numel()), float(beta), _ptr(a), _ptr(b),
                                    _stream(stream)), "qsvd_beta_exponents")


def qsvd_sq_diff_sum(y, yq, out, stream=None) -> None:
    """out[0] = sum (y - yq)^2 in float64 (device tensors; out float64)."""
    _check(_lib.qsvd_sq_diff_sum(_ptr(y), _ptr(yq), int(y.numel()), _ptr(out), _stream(stream)),
           "qsvd_sq_diff_sum")


def qsvd_prepare_per_head_fold(dims: qsvd_dims, bv, wo, f=None, stream=None) -> torch.Tensor:
    """F = [B_{Vh} W_{O,h}]_h (H r x E) in the weight type; returns F."""
    if f is None:
        f = torch.empty((dims.H * dims.r, dims.E), dtype=wo.dtype, device=wo.device)
    _check(_lib.qsvd_prepare_per_head_fold(ctypes.byref(dims), _ptr(bv), _ptr(wo), _ptr(f), _stream(stream)),
           "qsvd_prepare_per_head_fold")
    return f


def prefill_attention_workspace_bytes(dims: qsvd_dims) -> int:
    n = ctypes.c_size_t(0)
    _check(_lib.qsvd_prefill_attention(ctypes.byref(dims), None, None, None, None, ctypes.byref(n),
                                       None, None, None), "qsvd_prefill_attention(size)")
    return n.value


def qsvd_prefill_attention(dims: qsvd_dims, packed, cache, lengths, out, status, workspace=None,
                           stream=None):
    """Causal attention over the prompts' latent rows (cache rows b * max_len
    + t, t < lengths[b]); out is B x max_len x E.  Returns the workspace."""
    if workspace is None:
        workspace = _empty_bytes(prefill_attention_workspace_bytes(dims), cache.device)
    n = ctypes.c_size_t(workspace.numel() * workspace.element_size())
    _check(_lib.qsvd_prefill_attention(ctypes.byref(dims), _ptr(packed), _ptr(cache), _ptr(lengths),
                                       _ptr(workspace), ctypes.byref(n), _ptr(out), _ptr(status),
                                       _stream(stream)),
           "qsvd_prefill_attention")
    return workspace


def qsvd_append_latent_static(dims: qsvd_dims, packed, x, pos, cache, scales=None,
                              c_out=None, status=None, stream=None):
    """qsvd_append_latent for callers that cannot allocate: no workspace, the
    library's static device scratch instead (calls must not overlap)."""
    _check(_lib.qsvd_append_latent_static(ctypes.byref(dims), _ptr(packed), _ptr(x), _ptr(pos),
                                          _ptr(cache), _ptr(scales), _ptr(c_out), _ptr(status),
                                          _stream(stream)),
           "qsvd_append_latent_static")


def decode_workspace_bytes(dims: qsvd_dims, num_splits: int = 0) -> int:
    n = ctypes.c_size_t(0)
    _check(_lib.qsvd_decode_attn(ctypes.byref(dims), None, None, 1, None, None, None,
                                 int(num_splits), None, ctypes.byref(n), None, 0, None),
           "qsvd_decode_attn(size)")
    return n.value


def qsvd_decode_attn(dims: qsvd_dims, packed, qin, qin_is_latent, cache, scales, lengths,
                     out, num_splits=0, workspace=None, phases=0, stream=None):
    if workspace is None:
        workspace = _empty_bytes(decode_workspace_bytes(dims, num_splits), cache.device)
    n = ctypes.c_size_t(workspace.numel() * workspace.element_size())
    _check(_lib.qsvd_decode_attn(ctypes.byref(dims), _ptr(packed), _ptr(qin),
                                 int(bool(qin_is_latent)), _ptr(cache), _ptr(scales),
                                 _ptr(lengths), int(num_splits), _ptr(workspace),
                                 ctypes.byref(n), _ptr(out), int(phases), _stream(stream)),
           "qsvd_decode_attn")
    return workspace


def per_head_workspace_bytes(dims: qsvd_dims) -> int:
    n = ctypes.c_size_t(0)
    _check(_lib.qsvd_decode_attn_per_head(ctypes.byref(dims), None, None, None, None, None, None, 0, None,
                                          ctypes.byref(n), None, None),
           "qsvd_decode_attn_per_head(size)")
    return n.value


def qsvd_decode_attn_per_head(dims: qsvd_dims, bk, bv, q, ck, cv, lengths, out, workspace=None,
                              layout=QSVD_PER_HEAD_HEAD_MAJOR, stream=None):
    """Decode over per-head key/value latents (ck, cv: B x H x max_len x r,
    or B x max_len x H x r with layout QSVD_PER_HEAD_TOKEN_MAJOR); bk, bv:
    H x r x d_h; q: B x E float32.  Returns the workspace (its first int32
    is the status word)."""
    if workspace is None:
        workspace = _empty_bytes(per_head_workspace_bytes(dims), q.device)
    n = ctypes.c_size_t(workspace.numel() * workspace.element_size())
    _check(_lib.qsvd_decode_attn_per_head(ctypes.byref(dims), _ptr(bk), _ptr(bv), _ptr(q), _ptr(ck),
                                          _ptr(cv), _ptr(lengths), int(layout), _ptr(workspace), ctypes.byref(n),
                                          _ptr(out), _stream(stream)),
           "qsvd_decode_attn_per_head")
    return workspace


def qsvd_combine_splits(dims: qsvd_dims, packed, workspace, num_splits, lengths, out,
                        stream=None):
    _check(_lib.qsvd_combine_splits(ctypes.byref(dims), _ptr(packed), _ptr(workspace),
                                    int(num_splits), _ptr(lengths), _ptr(out), _stream(stream)),
           "qsvd_combine_splits")


def status_word(workspace: torch.Tensor) -> int:
    """Device status bits (QSVD_STATUS_*) recorded in a decode workspace."""
    return int(workspace[:4].view(torch.int32).item())


def exported_symbols():
    """Names of the C functions declared in include/qsvd.h."""
    return list(_sigs) + ["qsvd_status_string", "qsvd_last_error", "qsvd_kernel_launches",
                          "qsvd_abi_version"]
