"""Host-side checks of the per-head latent decode (qsvd_decode_attn_per_head),
no GPU: refusals, the workspace size, and the index arithmetic of its three
kernels replayed on the CPU for every CTA and thread of small and ragged
launches (every access inside its buffer, every valid token of every head
read exactly once, every chunk the merge reads written by the split).

The replay restates the kernels' index formulas (split_wsvd.cu); it checks
where they point, not what they compute.
"""
import ctypes

import numpy as np
import pytest

import rank_joint_qkv_b200 as q

CHUNK, T = 256, 128


def _dims(**kw):
    base = dict(E=512, H=4, d_h=128, r=64, batch=3, max_len=700)
    base.update(kw)
    opts = {k: base.pop(k) for k in list(base) if k not in ("E", "H", "d_h", "r", "batch", "max_len")}
    return q.make_dims(base["E"], base["H"], base["d_h"], base["r"], base["batch"], base["max_len"], **opts)


def _align(n):
    return (n + 255) // 256 * 256


def _layout(B, H, r, max_len, d_h=128):
    S = (max_len + CHUNK - 1) // CHUNK
    o = 0
    hdr = o; o = _align(o + 16)
    qt = o; o = _align(o + B * H * max(r, d_h) * 4)
    m = o; o = _align(o + B * H * S * 4)
    l_ = o; o = _align(o + B * H * S * 4)
    z = o; o = _align(o + B * H * S * r * 4)
    return dict(S=S, hdr=hdr, qt=qt, m=m, l=l_, z=z, total=o)


@pytest.mark.parametrize("shape", [dict(), dict(r=32, max_len=256), dict(r=96, max_len=1000),
                                   dict(r=256, batch=1, max_len=5000)])
def test_workspace_size_matches_layout(shape):
    d = _dims(**shape)
    want = _layout(d.batch, d.H, d.r, d.max_len)["total"]
    assert q.per_head_workspace_bytes(d) == want


@pytest.mark.parametrize("bad,status", [(dict(rope=True, r=96), q.QSVD_ERR_UNSUPPORTED),
                                        (dict(rope=True, cache="f32"), q.QSVD_ERR_UNSUPPORTED),
                                        (dict(rope=True, cache="bf16"), q.QSVD_ERR_UNSUPPORTED),
                                        (dict(rope=True, E=60 * 128, H=60), q.QSVD_ERR_UNSUPPORTED),
                                        (dict(cache="i4", r=128), q.QSVD_ERR_UNSUPPORTED),
                                        (dict(out_proj="chain"), q.QSVD_ERR_UNSUPPORTED),
                                        (dict(out_proj="fold", weight="f32"), q.QSVD_ERR_UNSUPPORTED),
                                        (dict(h2=True, h2_m=2), q.QSVD_ERR_UNSUPPORTED),
                                        (dict(r=48), q.QSVD_ERR_INVALID_ARG)])
def test_refusals_on_host(bad, status):
    with pytest.raises(q.QsvdError) as e:
        q.per_head_workspace_bytes(_dims(**bad))
    assert e.value.status == status


def test_null_pointers_and_small_workspace():
    d = _dims()
    n = ctypes.c_size_t(64)
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: the checks fail first
    st = q._lib.qsvd_decode_attn_per_head(ctypes.byref(d), fake, fake, fake, fake, fake, fake, 0, fake,
                                          ctypes.byref(n), fake, None)
    assert st == q.QSVD_ERR_WORKSPACE
    n = ctypes.c_size_t(1 << 30)
    st = q._lib.qsvd_decode_attn_per_head(ctypes.byref(d), None, fake, fake, fake, fake, fake, 0, fake,
                                          ctypes.byref(n), fake, None)
    assert st == q.QSVD_ERR_INVALID_ARG
    st = q._lib.qsvd_decode_attn_per_head(ctypes.byref(d), fake, fake, fake, fake, fake, fake, 2, None,
                                          ctypes.byref(n), fake, None)
    assert st == q.QSVD_ERR_INVALID_ARG and b"layout" in q._lib.qsvd_last_error()


def _replay(B, H, d_h, r, max_len, lengths, token_major=False):
    """Replay the three launches' index arithmetic; return the read counts
    of every latent row (b, h, t)."""
    E = H * d_h
    W = _layout(B, H, r, max_len)
    S = W["S"]
    n_cache = B * H * max_len * r
    rows_read = np.zeros((B, H, max_len), np.int64)
    written = np.zeros(B * H * S, bool)
    # absorb: grid (H, B); q reads and qt writes
    for b in range(B):
        for h in range(H):
            qrow = (b * H + h) * d_h
            assert 0 <= qrow and qrow + d_h <= B * E
            assert (b * H + h) * r + r <= B * H * r
            assert h * r * d_h + r * d_h <= H * r * d_h          # B_K rows of head h
    # split: grid (S, H, B)
    ng = T // r if (r < T and T % r == 0) else 1
    smem = r + CHUNK + 4 + ng * r
    assert ng * r <= max(r, T)
    for b in range(B):
        ln = min(max(int(lengths[b]), 0), max_len)
        for h in range(H):
            for sp in range(S):
                t0 = sp * CHUNK
                if t0 >= ln:
                    continue
                n = min(CHUNK, ln - t0)
                bh = b * H + h
                row0 = (b * max_len + t0) * H + h if token_major else bh * max_len + t0
                rs = H * r if token_major else r
                kb = row0 * r
                for t in range(n):                         # score rows (warp per row)
                    lo, hi = kb + t * rs, kb + t * rs + r
                    assert 0 <= lo and hi <= n_cache
                    # the row this is in the caller's layout
                    want = ((b * max_len + t0 + t) * H + h) * r if token_major else \
                        ((b * H + h) * max_len + t0 + t) * r
                    assert lo == want
                    rows_read[b, h, t0 + t] += 1
                assert n <= CHUNK                           # ss[t] inside its section
                if ng > 1:                                  # value rows by token groups
                    for tid in range(T):
                        g, j = tid // r, tid % r
                        assert g * r + j < ng * r
                        for t in range(g, n, ng):
                            assert kb + t * rs + j < n_cache
                slot = bh * S + sp
                assert slot < B * H * S and (slot + 1) * r <= B * H * S * r
                written[slot] = True
    # combine: grid (H, B); reads the chunks s < ceil(len / CHUNK)
    for b in range(B):
        ln = min(max(int(lengths[b]), 0), max_len)
        su = (ln + CHUNK - 1) // CHUNK
        assert su <= S and S + r + 4 <= 227 * 1024 // 4
        for h in range(H):
            base = (b * H + h) * S
            for s in range(su):
                assert written[base + s]
            assert (b * H + h) * d_h + d_h <= B * E             # output row
    return rows_read, smem


@pytest.mark.parametrize("B,H,d_h,r,max_len,lengths", [
    (3, 4, 128, 64, 700, [700, 1, 300]),
    (2, 2, 64, 32, 256, [256, 255]),
    (2, 3, 128, 96, 513, [513, 0]),
    (1, 2, 128, 256, 1000, [777]),
    (2, 2, 64, 128, 300, [-5, 9999]),                      # clamped to 0 and max_len
])
@pytest.mark.parametrize("token_major", [False, True])
def test_index_replay(B, H, d_h, r, max_len, lengths, token_major):
    rows, smem = _replay(B, H, d_h, r, max_len, lengths, token_major)
    for b in range(B):
        ln = min(max(lengths[b], 0), max_len)
        assert np.all(rows[b, :, :ln] == 1) and np.all(rows[b, :, ln:] == 0)
    assert smem * 4 <= 227 * 1024


def _replay_vec(B, H, r, max_len, lengths, token_major):
    """The 16-byte-vector split kernel (16-bit latents, r in {64, 128, 256}):
    grid (S, H, B), 256 threads; thread (vj = tid % (r / 8), tg = tid // (r / 8))
    reads vector vj of rows t = p * (256 / (r / 8)) + tg.  Returns how often
    each element of the cache is read (keys; the value side is identical)."""
    TPR = r // 8
    TPP = 256 // TPR
    NP = CHUNK // TPP
    assert NP * TPP == CHUNK
    S = (max_len + CHUNK - 1) // CHUNK
    n_cache = B * H * max_len * r
    hits = np.zeros(n_cache, np.int64)
    for b in range(B):
        ln = min(max(int(lengths[b]), 0), max_len)
        for h in range(H):
            for sp in range(S):
                t0 = sp * CHUNK
                if t0 >= ln:
                    continue
                n = min(CHUNK, ln - t0)
                row0 = (b * max_len + t0) * H + h if token_major else (b * H + h) * max_len + t0
                rsv = (H * r if token_major else r) // 8
                for tid in range(256):
                    vj, tg = tid % TPR, tid // TPR
                    assert tg < TPP and 8 * vj + 7 < r            # zr[tg][8 vj + e]
                    for p in range(NP):
                        t = p * TPP + tg
                        assert t < CHUNK                            # ss[t]
                        if t >= n:
                            continue
                        v = row0 * r // 8 + vj + t * rsv            # 16-byte vector index
                        assert (row0 * r) % 8 == 0
                        lo = 8 * v
                        assert 0 <= lo and lo + 8 <= n_cache
                        hits[lo:lo + 8] += 1
    return hits


@pytest.mark.parametrize("B,H,r,max_len,lengths", [
    (3, 4, 64, 700, [700, 1, 300]),
    (2, 2, 128, 513, [513, 0]),
    (1, 2, 256, 1000, [777]),
    (2, 2, 64, 300, [-5, 9999]),
])
@pytest.mark.parametrize("token_major", [False, True])
def test_vector_split_index_replay(B, H, r, max_len, lengths, token_major):
    hits = _replay_vec(B, H, r, max_len, lengths, token_major)
    want = np.zeros((B, max_len, H, r) if token_major else (B, H, max_len, r), np.int64)
    for b in range(B):
        ln = min(max(lengths[b], 0), max_len)
        if token_major:
            want[b, :ln] = 1
        else:
            want[b, :, :ln] = 1
    assert np.array_equal(hits, want.reshape(-1))    # every valid element once, nothing else


@pytest.mark.parametrize("r", [64, 128])
@pytest.mark.parametrize("H", [1, 32, 40, 59])
def test_rotary_scores_shared_memory_map(r, H):
    """k_wsvd_rope_scores' shared memory (wsvd_rope.cu), restated: the load
    stages, the staged cos/sin rows (128 x 130 floats), 128 bytes of
    barriers (full / empty per stage, done / tfree per TMEM buffer, drain,
    the TMEM address, the abort flag) and every head's rotated query
    (H x 128 floats): disjoint and aligned inside the launch's dynamic size
    (whose base is aligned up by at most 1023 bytes), and with the static
    partial dots (3 x 2 x 128 floats) within the 227 KB per block."""
    nst = 4 if r == 64 else 2
    stage = 128 * r * 2 + r * 128 * 2
    tab = nst * stage                       # offsets from the 1024-aligned base
    bars = tab + 128 * 130 * 4
    nbar = 2 * nst + 5
    holder = bars + 8 * nbar
    abort = holder + 4
    qsm = bars + 128
    assert stage % 1024 == 0 and tab % 1024 == 0          # swizzled TMA boxes
    assert bars % 8 == 0 and abort + 4 <= qsm             # barriers inside their 128 bytes
    assert qsm % 16 == 0
    end = qsm + H * 128 * 4
    dynamic = 1024 + nst * stage + 128 * 130 * 4 + 128 + H * 128 * 4   # the launch's size
    assert end + 1023 <= dynamic
    assert dynamic + 3 * 2 * 128 * 4 <= 232448


def test_rotary_rows_beyond_32_bit_coordinates_are_refused():
    """Head-major rows (b H + h) max_len + t are tensor-map coordinates of
    the rotary scores kernel: B x H x max_len must stay below 2^31."""
    ok = _dims(rope=True, E=32 * 128, H=32, batch=(1 << 11) - 1, max_len=1 << 15)
    assert q.per_head_workspace_bytes(ok) > 0
    bad = _dims(rope=True, E=32 * 128, H=32, batch=1 << 11, max_len=1 << 15)
    with pytest.raises(q.QsvdError) as e:
        q.per_head_workspace_bytes(bad)
    assert e.value.status == q.QSVD_ERR_UNSUPPORTED
    assert b"2^31" in q._lib.qsvd_last_error()
