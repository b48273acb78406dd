"""C-ABI checks that need no GPU: the library loads, exports every function
declared in include/qsvd.h, agrees with the header on the struct layout, and
rejects invalid arguments on the host before touching the device."""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest

import rank_joint_qkv_b200 as q

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qsvd.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(qsvd_[a-z_]+)\s*\(", src)))


def test_header_declares_the_four_calls():
    names = declared_functions()
    for n in ("qsvd_prepare_weights", "qsvd_append_latent", "qsvd_decode_attn",
              "qsvd_combine_splits"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(q.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing
    assert sorted(q.exported_symbols()) == declared_functions()


def test_abi_version_matches_header():
    m = re.search(r"#define QSVD_ABI_VERSION (\d+)", open(HEADER).read())
    assert q.abi_version() == int(m.group(1))


def test_struct_layout_matches_header():
    """Compile a C probe against the header; compare sizeof/offsetof."""
    fields = [f for f, _ in q.qsvd_dims._fields_]
    body = "\n".join(f'printf("%zu ", offsetof(qsvd_dims, {f}));' for f in fields)
    prog = f"""
#include <stdio.h>
#include <stddef.h>
#include "qsvd.h"
int main(void) {{ printf("%zu ", sizeof(qsvd_dims)); {body} return 0; }}
"""
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "p.c")
        open(c, "w").write(prog)
        exe = os.path.join(d, "p")
        subprocess.run(["gcc", "-I", os.path.dirname(HEADER), c, "-o", exe], check=True)
        got = list(map(int, subprocess.run([exe], capture_output=True, text=True,
                                           check=True).stdout.split()))
    want = [ctypes.sizeof(q.qsvd_dims)] + [getattr(q.qsvd_dims, f).offset for f in fields]
    assert got == want


def _dims(**kw):
    base = dict(E=512, H=4, d_h=128, r=256, batch=2, max_len=300)
    base.update(kw)
    opts = {k: base.pop(k) for k in list(base) if k not in ("E", "H", "d_h", "r", "batch", "max_len")}
    return q.make_dims(base["E"], base["H"], base["d_h"], base["r"], base["batch"],
                       base["max_len"], **opts)


@pytest.mark.parametrize("bad", [
    dict(E=500), dict(H=3), dict(r=100), dict(r=16), dict(batch=0), dict(max_len=0),
    dict(cache="i4", group=100), dict(cache="i8", group=96), dict(d_h=130, E=520),
    dict(h2=True, h2_m=3),                   # r/h2_m = 256/3 not an integer
    dict(H=(1 << 24) + 1, d_h=256, E=256),   # H d_h wraps to E in 32-bit arithmetic
    dict(batch=1 << 15, max_len=1 << 16),    # 2^31 cache rows: beyond 32-bit coordinates
    dict(batch=65536, max_len=16),           # sequences beyond a grid's y / z extent
])
def test_invalid_dims_rejected_on_host(bad):
    d = _dims(**bad)
    with pytest.raises(q.QsvdError) as e:
        q.decode_workspace_bytes(d, num_splits=4)
    assert e.value.status == q.QSVD_ERR_INVALID_ARG


def test_rope_needs_d_h_multiple_of_64():
    d = _dims(E=384, H=4, d_h=96, rope=True)
    with pytest.raises(q.QsvdError) as e:
        q.decode_workspace_bytes(d, num_splits=4)
    assert e.value.status == q.QSVD_ERR_UNSUPPORTED


def test_workspace_query_on_host():
    d = _dims(max_len=3000)
    n4 = q.decode_workspace_bytes(d, num_splits=4)
    n8 = q.decode_workspace_bytes(d, num_splits=8)
    # 4 more partial slots of H x r latent floats (m, l sections are padded)
    assert n8 - n4 >= 4 * 4 * 256 * 4
    assert n4 % 256 == 0
    # splits beyond the number of 128-token tiles are not used
    d2 = _dims(max_len=300)
    assert q.decode_workspace_bytes(d2, num_splits=6) == q.decode_workspace_bytes(d2, num_splits=60)
    assert q.append_workspace_bytes(d) > 0


def _split_begin(c, G, T):
    return (c * T) // G


def _split_of_tile(t, G, T):
    return ((t + 1) * G - 1) // T


def test_split_count_is_capped_where_a_sequence_could_span_more_merge_weights():
    """Tiles of all sequences are dealt to G splits in equal contiguous runs
    (internal.cuh split_begin / split_of_tile, restated).  When G exceeds
    the tiles present at run time, empty splits lie between a sequence's
    tiles, and its run of split indices c0..c1 (one merge weight each, held
    in shared memory) grows towards G, far past its tile count.  The host
    caps G at 2048, the merge's capacity."""
    lens = [2047] + [1] * 15                      # tiles per sequence
    T, G = sum(lens), 16 * 2047                   # G = B x tiles(max_len)
    t0 = 0
    for k in lens:
        c0, c1 = _split_of_tile(t0, G, T), _split_of_tile(t0 + k - 1, G, T)
        assert _split_begin(c0, G, T) <= t0 < _split_begin(c0 + 1, G, T)
        assert c1 - c0 + 1 <= G
        if k == 2047:
            assert c1 - c0 + 1 > 2048             # what an uncapped G would meet
        t0 += k
    for G in (1, 7, 148, 2048):                   # the run never exceeds G
        t0 = 0
        for k in lens:
            c0, c1 = _split_of_tile(t0, G, T), _split_of_tile(t0 + k - 1, G, T)
            assert 1 <= c1 - c0 + 1 <= min(G, k + 1)
            t0 += k
    d = _dims(max_len=2047 * 128)
    d.batch = 16
    assert q.decode_workspace_bytes(d, num_splits=4096) == q.decode_workspace_bytes(d, num_splits=2048)
    assert q.decode_workspace_bytes(d, num_splits=2047) < q.decode_workspace_bytes(d, num_splits=2048)


def test_too_small_workspace_and_null_pointers():
    lib = ctypes.CDLL(q.LIB_PATH)
    lib.qsvd_decode_attn.argtypes = q._sigs["qsvd_decode_attn"]
    d = _dims()
    n = ctypes.c_size_t(16)
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the size check fails first
    st = lib.qsvd_decode_attn(ctypes.byref(d), fake, fake, 1, fake, None, fake, 4, fake,
                              ctypes.byref(n), fake, 0, None)
    assert st == q.QSVD_ERR_WORKSPACE
    n = ctypes.c_size_t(1 << 40)
    st = lib.qsvd_decode_attn(ctypes.byref(d), None, fake, 1, fake, None, fake, 4, fake,
                              ctypes.byref(n), fake, 0, None)
    assert st == q.QSVD_ERR_INVALID_ARG
    assert b"NULL" in q._lib.qsvd_last_error()


def test_status_strings():
    for s in range(5):
        assert q._lib.qsvd_status_string(s).startswith(b"QSVD_")


def test_header_constants_match_binding():
    """Every QSVD_PHASE_ / QSVD_STATUS_ / QSVD_KERNEL_ value of the header
    has the same value in the Python binding."""
    src = open(HEADER).read()
    consts = dict(re.findall(r"#define (QSVD_(?:PHASE|STATUS|KERNEL|OUT_PROJ)_[A-Z0-9_]+) (\d+)u?", src))
    assert "QSVD_OUT_PROJ_FOLD" in consts
    assert any(k.startswith("QSVD_PHASE_SPLIT_") for k in consts)
    assert "QSVD_KERNEL_TCGEN05" in consts
    for name, val in consts.items():
        assert getattr(q, name) == int(val), name


def test_split_sub_phases_rejected_outside_rotary_tensor_path():
    """The sub-phase bits are refused on the host for the absorbed path and
    for the rotary CUDA-core path (before the device is touched)."""
    lib = ctypes.CDLL(q.LIB_PATH)
    lib.qsvd_decode_attn.argtypes = q._sigs["qsvd_decode_attn"]
    fake = ctypes.c_void_p(1 << 20)
    for d in (_dims(), _dims(rope=True, kernel=q.QSVD_KERNEL_SIMT)):
        for ph in (q.QSVD_PHASE_SPLIT_SCORES, q.QSVD_PHASE_SPLIT_ACCUM):
            n = ctypes.c_size_t(1 << 40)
            st = lib.qsvd_decode_attn(ctypes.byref(d), fake, fake, 1, fake, None, fake, 4, fake,
                                      ctypes.byref(n), fake, ph, None)
            assert st == q.QSVD_ERR_INVALID_ARG
            assert b"sub-phases" in q._lib.qsvd_last_error()
    n = ctypes.c_size_t(1 << 40)
    st = lib.qsvd_decode_attn(ctypes.byref(_dims()), fake, fake, 1, fake, None, fake, 4, fake,
                              ctypes.byref(n), fake, 32, None)
    assert st == q.QSVD_ERR_INVALID_ARG


@pytest.mark.parametrize("bad", [dict(cache="i4"), dict(rope=True), dict(H=40, E=5120),
                                 dict(r=64 * 3, E=512), dict(r=128 * 9 * 2, E=2304, H=18)])
def test_cluster_kernel_refused_where_it_does_not_apply(bad):
    """Forcing the cluster kernel on dims it does not cover is UNSUPPORTED,
    decided on the host."""
    d = _dims(kernel=q.QSVD_KERNEL_TCGEN05_CLUSTER, **bad)
    with pytest.raises(q.QsvdError) as e:
        q.decode_workspace_bytes(d, num_splits=4)
    assert e.value.status == q.QSVD_ERR_UNSUPPORTED


@pytest.mark.parametrize("bad", [dict(weight="f32", cache="f32"), dict(r=384, E=512),
                                 dict(h2=True, h2_m=2), dict(cache="i4", group=64)])
def test_prefill_refused_where_it_does_not_apply(bad):
    """qsvd_prefill_latent: dims it has no kernel for are UNSUPPORTED, on the
    host, before any pointer is looked at."""
    lib = ctypes.CDLL(q.LIB_PATH)
    lib.qsvd_prefill_latent.argtypes = q._sigs["qsvd_prefill_latent"]
    d = _dims(**bad)
    fake = ctypes.c_void_p(1 << 20)
    st = lib.qsvd_prefill_latent(ctypes.byref(d), fake, fake, 4, fake, fake, fake, None, None, None)
    assert st == q.QSVD_ERR_UNSUPPORTED, q._lib.qsvd_last_error()


def test_prefill_row_count_checked_on_host():
    lib = ctypes.CDLL(q.LIB_PATH)
    lib.qsvd_prefill_latent.argtypes = q._sigs["qsvd_prefill_latent"]
    d = _dims()
    st = lib.qsvd_prefill_latent(ctypes.byref(d), None, None, -1, None, None, None, None, None, None)
    assert st == q.QSVD_ERR_INVALID_ARG
    # no rows: nothing to do, no pointer needed
    st = lib.qsvd_prefill_latent(ctypes.byref(d), None, None, 0, None, None, None, None, None, None)
    assert st == q.QSVD_OK


def _packed_bytes(d):
    n = ctypes.c_size_t(0)
    st = q._lib.qsvd_prepare_weights(ctypes.byref(d), None, None, None, None, None, None,
                                     ctypes.byref(n), None)
    assert st == q.QSVD_OK
    return n.value


def test_out_proj_sections_sized_on_host():
    """The packed buffer gains W_O (E x E) for the chain and F (H r x E) for
    the fold; the decode workspace gains the projection's partials."""
    base = _packed_bytes(_dims())
    E, H, r = 512, 4, 256
    assert _packed_bytes(_dims(out_proj="chain")) == base + E * E * 2
    assert _packed_bytes(_dims(out_proj="fold")) == base + H * r * E * 2
    w0 = q.decode_workspace_bytes(_dims(), num_splits=4)
    # chain: o (B x E fp32) + ceil(E/512) partials of B x E
    assert q.decode_workspace_bytes(_dims(out_proj="chain"), num_splits=4) >= w0 + 2 * 512 * 4 * 2
    # fold: ceil(H r / 512) = 2 partials of B x E
    assert q.decode_workspace_bytes(_dims(out_proj="fold"), num_splits=4) >= w0 + 2 * 2 * 512 * 4


def test_out_proj_refused_on_host():
    d = _dims()
    d.out_proj = 3
    with pytest.raises(q.QsvdError) as e:
        q.decode_workspace_bytes(d, num_splits=4)
    assert e.value.status == q.QSVD_ERR_INVALID_ARG
    # fp32 weights have no tensor-core GEMV: the projection is UNSUPPORTED
    d = _dims(weight="f32", cache="f32", out_proj="fold")
    with pytest.raises(q.QsvdError) as e:
        q.decode_workspace_bytes(d, num_splits=4)
    assert e.value.status == q.QSVD_ERR_UNSUPPORTED
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: the checks fail first
    assert q._lib.qsvd_prepare_out_proj(ctypes.byref(d), fake, fake, 1 << 30, None) == \
        q.QSVD_ERR_UNSUPPORTED
    d = _dims()
    assert q._lib.qsvd_prepare_out_proj(ctypes.byref(d), fake, fake, 1 << 30, None) == \
        q.QSVD_ERR_INVALID_ARG
    d = _dims(out_proj="chain")
    assert q._lib.qsvd_prepare_out_proj(ctypes.byref(d), fake, fake, 256, None) == \
        q.QSVD_ERR_WORKSPACE


def test_split_factors_pointers_checked_on_host():
    d = _dims()
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: the NULL check fails first
    st = q._lib.qsvd_split_factors(ctypes.byref(d), fake, fake, fake, None, fake, fake, fake, fake, None)
    assert st == q.QSVD_ERR_INVALID_ARG
    assert b"NULL" in q._lib.qsvd_last_error()


def test_prefill_attention_host_checks():
    """Workspace size and refusals of qsvd_prefill_attention, no GPU."""
    d = q.make_dims(512, 4, 128, 256, 3, 305, cache="f16", weight="f16")
    n = 3 * 305
    al = lambda x: (x + 255) // 256 * 256
    want = al(n * 512 * 4) + 6 * al(n * 512 * 2)
    assert q.prefill_attention_workspace_bytes(d) == want
    for bad in (q.make_dims(512, 8, 64, 256, 3, 305, cache="f16", weight="f16"),      # d_h 64
                q.make_dims(512, 4, 128, 256, 3, 305, cache="i4", weight="f16"),      # int cache
                q.make_dims(512, 4, 128, 256, 3, 305, cache="bf16", weight="f16"),    # mixed types
                q.make_dims(640, 5, 128, 256, 3, 305, cache="f16", weight="f16")):    # E % 256
        with pytest.raises(q.QsvdError) as e:
            q.prefill_attention_workspace_bytes(bad)
        assert e.value.status == q.QSVD_ERR_UNSUPPORTED


def test_misaligned_outputs_and_scales_are_refused():
    """The decode's fp32 output is stored as float4 and the fp16 group scales
    two bytes at a time: pointers off those boundaries are refused on the
    host, before anything is enqueued (the pointers are never dereferenced)."""
    lib = ctypes.CDLL(q.LIB_PATH)
    for name in ("qsvd_decode_attn", "qsvd_append_latent", "qsvd_decode_attn_per_head",
                 "qsvd_prefill_latent"):
        getattr(lib, name).argtypes = q._sigs[name]
    fake = ctypes.c_void_p(1 << 20)
    odd, off8 = ctypes.c_void_p((1 << 20) + 1), ctypes.c_void_p((1 << 20) + 8)
    n = ctypes.c_size_t(1 << 40)
    st = lib.qsvd_decode_attn(ctypes.byref(_dims()), fake, fake, 1, fake, None, fake, 4, fake,
                              ctypes.byref(n), off8, 0, None)
    assert st == q.QSVD_ERR_INVALID_ARG and b"out must be 16-byte" in q._lib.qsvd_last_error()
    st = lib.qsvd_decode_attn(ctypes.byref(_dims(cache="i8")), fake, fake, 1, fake, odd, fake, 4, fake,
                              ctypes.byref(n), fake, 0, None)
    assert st == q.QSVD_ERR_INVALID_ARG and b"scales 2-byte" in q._lib.qsvd_last_error()
    st = lib.qsvd_append_latent(ctypes.byref(_dims(cache="i8")), fake, fake, fake, fake, odd, fake, None,
                                fake, ctypes.byref(n), None)
    assert st == q.QSVD_ERR_INVALID_ARG and b"scales must be 2-byte" in q._lib.qsvd_last_error()
    d = _dims(cache="i8", weight="f16")
    st = lib.qsvd_prefill_latent(ctypes.byref(d), fake, fake, 4, fake, fake, odd, None, None, None)
    assert st == q.QSVD_ERR_INVALID_ARG and b"scales must be 2-byte" in q._lib.qsvd_last_error()
    dh = q.make_dims(512, 4, 128, 64, 3, 700, cache="f16", weight="f16")
    st = lib.qsvd_decode_attn_per_head(ctypes.byref(dh), fake, fake, fake, fake, fake, fake, 0, fake,
                                       ctypes.byref(n), off8, None)
    assert st == q.QSVD_ERR_INVALID_ARG and b"out must be 16-byte" in q._lib.qsvd_last_error()


def _prototypes():
    """name -> (return type, [parameter types]) of every call in the header."""
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    out = {}
    for m in re.finditer(r"([A-Za-z_][A-Za-z0-9_ \*]*?)\b(qsvd_[a-z_]+)\s*\(([^)]*)\)\s*;", src):
        params = [" ".join(p.split()) for p in m.group(3).split(",")]
        params = [] if params == ["void"] else [p.rsplit(" ", 1)[0] if not p.endswith("*") else p
                                                for p in params]
        out[m.group(2)] = (" ".join(m.group(1).split()), params)
    return out


def _ctype_of(param):
    """The ctypes type a parameter of this C type must be declared with."""
    t = param.replace("const ", "").strip()
    if t.startswith("qsvd_dims"):
        return ctypes.POINTER(q.qsvd_dims)
    if t.startswith("size_t") and "*" in t:
        return ctypes.POINTER(ctypes.c_size_t)
    if "*" in t:
        return ctypes.c_void_p
    return {"int": ctypes.c_int, "unsigned": ctypes.c_uint, "size_t": ctypes.c_size_t,
            "double": ctypes.c_double, "int64_t": ctypes.c_int64,
            "unsigned long long": ctypes.c_ulonglong, "qsvd_status": ctypes.c_int}[t]


def test_binding_signatures_match_the_header():
    """Every call's ctypes argtypes have the header's parameter count and
    types (a pointer as c_void_p, size_t* and qsvd_dims* as typed
    pointers), so no argument is dropped, narrowed or widened on the way."""
    protos = _prototypes()
    assert set(q._sigs) | {"qsvd_status_string", "qsvd_last_error", "qsvd_kernel_launches",
                           "qsvd_abi_version"} == set(protos)
    for name, args in q._sigs.items():
        ret, params = protos[name]
        assert ret == "qsvd_status", name
        assert len(args) == len(params), f"{name}: {len(args)} argtypes, header has {len(params)}"
        for i, (a, p) in enumerate(zip(args, params)):
            want = _ctype_of(p)
            assert a is want or (hasattr(a, "_type_") and hasattr(want, "_type_") and a._type_ is want._type_
                                 and a.__name__ == want.__name__), f"{name} argument {i}: {p!r}"
    # pointer-sized and 64-bit results keep their width
    assert q._lib.qsvd_last_error.restype is ctypes.c_char_p
    assert q._lib.qsvd_status_string.restype is ctypes.c_char_p
    assert q._lib.qsvd_kernel_launches.restype is ctypes.c_uint64
