"""Host-side replay of the quantised split kernel's shared-memory index
arithmetic (split_tc.cu), no GPU.

The kernel expands a Z item of int8 / int4 codes in place: the raw codes
(64 rows x 128 channels) land at the end of the item's 16 KB fp16 slot and a
warp rewrites the slot as two 128-byte-swizzled boxes of 64 rows x 64 fp16
channels, in two phases of 32 rows.  These tests restate the converter's
formulas (convert_z_inplace) and check where they point, not what they
compute: every raw byte is read once, every byte of the slot is written
once, every access stays inside the slot, and no store lands on a raw byte
before the phase that reads it has loaded it.  The int4 unpack of S items
(unpack_s_group) and the 128-byte swizzle are checked the same way.
"""
import pytest

Z_SLOT = 16384          # kZSlotBytes: 64 tokens x 128 channels x 2 bytes
Z_BOX = 8192            # kZBoxBytes: one 64-channel box of 64 rows


def _z_phase_accesses(qb):
    """Per phase: (bytes loaded, bytes stored) of one converting warp, as the
    kernel's formulas give them (32 lanes, NV vectors per lane)."""
    rpb = qb * 16                 # raw bytes per row
    vpr = rpb // 16               # 16-byte vectors per row
    cpv = 4 if qb == 4 else 2     # 16-byte fp16 chunks per vector
    nv = 32 * vpr // 32           # vectors per lane per phase
    raw = Z_SLOT - 64 * rpb
    phases = []
    for ph in range(2):
        loads, stores = [], []
        for lane in range(32):
            for i in range(nv):
                v = lane + 32 * i
                tt, q = 32 * ph + v // vpr, v % vpr
                loads.append(raw + tt * rpb + q * 16)
                ch = q * (cpv * 8)
                box, c0 = ch >> 6, (ch & 63) >> 3
                for c in range(cpv):
                    stores.append(box * Z_BOX + tt * 128 + (((c0 + c) ^ (tt & 7)) << 4))
        phases.append((loads, stores))
    return raw, phases


@pytest.mark.parametrize("qb", [4, 8])
def test_in_place_z_expansion_reads_before_it_overwrites(qb):
    raw, phases = _z_phase_accesses(qb)
    read = {}
    for ph, (loads, _) in enumerate(phases):
        for a in loads:
            for x in range(a, a + 16):
                assert x not in read, "a raw byte is read twice"
                read[x] = ph
    assert sorted(read) == list(range(raw, Z_SLOT)), "the raw codes are read exactly once"
    written = set()
    for ph, (_, stores) in enumerate(phases):
        for a in stores:
            assert 0 <= a and a + 16 <= Z_SLOT
            for x in range(a, a + 16):
                assert x not in written, "a slot byte is written twice"
                written.add(x)
                if x in read:
                    assert read[x] <= ph, "a store lands on raw codes a later phase still reads"
    assert written == set(range(Z_SLOT)), "the fp16 item fills its slot"


@pytest.mark.parametrize("qb", [4, 8])
def test_z_stores_follow_the_128_byte_swizzle(qb):
    """Row tt of a box is 128 bytes; its 16-byte chunk c sits at c ^ (tt & 7):
    within each (box, row) the eight chunks are a permutation of 0..7."""
    _, phases = _z_phase_accesses(qb)
    rows = {}
    for _, stores in phases:
        for a in stores:
            box, rest = divmod(a, Z_BOX)
            tt, within = divmod(rest, 128)
            rows.setdefault((box, tt), []).append(within // 16)
    assert len(rows) == 2 * 64
    assert all(sorted(v) == list(range(8)) for v in rows.values())


def test_int4_s_unpack_covers_the_a_operand_once():
    """unpack_s_group: raw [128 rows][64 bytes] -> [128 rows][128 bytes]
    K-major, 128-byte swizzled; 16 vectors per lane, two stores each."""
    reads, writes = set(), set()
    for half in range(2):
        for lane in range(32):
            for i in range(8):
                v = lane + 32 * (8 * half + i)
                for x in range(v * 16, v * 16 + 16):
                    assert x not in reads
                    reads.add(x)
                t, c0 = v >> 2, 2 * (v & 3)
                for c in (c0, c0 + 1):
                    a = t * 128 + ((c ^ (t & 7)) << 4)
                    for x in range(a, a + 16):
                        assert x not in writes
                        writes.add(x)
    assert reads == set(range(128 * 64))
    assert writes == set(range(128 * 128))


@pytest.mark.parametrize("np_,r", [(32, 768), (16, 1536), (32, 1664), (16, 3712)])
def test_quantised_shared_memory_budget(np_, r):
    """The launch's sizing (launch_t, quantised latent): S slots of codes +
    query parts, the int4 raw ring, three scale tables of 128 x r/128 fp16,
    fp16 Z slots; at least 4 Z slots and the whole within 227 KB."""
    k_smem, misc, max_slots = 232448, 2048, 8
    pbuf = 2 * np_ * 128
    sq = 128 * 128 + 3 * np_ * 128
    for qb in (4, 8):
        nraw = 4 if qb == 4 else 0
        raw_s = 128 * 64 if qb == 4 else 0
        tables = 3 * 256 * (r // 128)
        avail = k_smem - 1024 - misc - 2 * pbuf - tables - nraw * raw_s
        for ns in ((2,) if qb == 4 else (3, 2)):
            nz = (avail - ns * sq) // Z_SLOT
            if nz >= 5:
                break
        nz = min(nz, max_slots)
        assert nz >= 4
        smem = 1024 + ns * sq + nz * Z_SLOT + 2 * pbuf + nraw * raw_s + tables + misc
        assert smem <= k_smem


@pytest.mark.parametrize("np_,ps,qb,r", [(32, 1, 0, 1536), (16, 1, 0, 512), (32, 2, 0, 1536), (16, 2, 0, 384),
                                          (32, 1, 8, 768), (32, 1, 4, 768), (16, 1, 8, 384),
                                          (32, 1, 8, 1536), (32, 1, 4, 1664), (16, 1, 4, 3712)])
def test_split_kernel_shared_memory_carve(np_, ps, qb, r):
    """carve() and the launch's size (split_tc.cu), restated for the 16-bit
    (qb 0) and quantised paths: slot rings and P buffers on 1024-byte
    boundaries (128-byte-swizzled TMA boxes and MMA operands), the barrier
    area (80 barriers, 71 used) and the misc region after them, the whole
    within the launched size and 227 KB."""
    k_smem, misc, max_slots, z_slot = 232448, 2048, 8, 16384
    pbuf = 2 * np_ * 128
    if qb == 0:
        a_slot = 128 * 128 + 2 * np_ * 128               # latent box + hi/lo query box
        avail = k_smem - 1024 - misc - 2 * ps * pbuf
        ns = min(96 * 1024 // a_slot, max_slots)
        nz = min((avail - ns * a_slot) // z_slot, max_slots)
        nraw, raw_s, tables = 0, 0, 0
    else:
        a_slot = 128 * 128 + 3 * np_ * 128               # codes + int8 query parts
        nraw, raw_s = (4, 128 * 64) if qb == 4 else (0, 0)
        tables = 3 * 256 * (r // 128)
        avail = k_smem - 1024 - misc - 2 * ps * pbuf - tables - nraw * raw_s
        for ns in ((2,) if qb == 4 else (3, 2)):
            nz = (avail - ns * a_slot) // z_slot
            if nz >= 5:
                break
        nz = min(nz, max_slots)
    zring = ns * a_slot
    pb = zring + nz * z_slot
    sraw = pb + 2 * ps * pbuf
    zsc = sraw + nraw * raw_s
    m = zsc + tables
    assert a_slot % 1024 == 0 and zring % 1024 == 0 and pb % 1024 == 0
    assert sraw % 1024 == 0 and zsc % 16 == 0 and m % 8 == 0
    nbar = 4 * max_slots + 8 + 2 * 4 + 8 + max_slots + 1 + 2 * 3
    assert nbar == 71 and nbar * 8 <= 640
    misc_used = 640 + 4 * np_ * 4 + 32 + (4 if qb else 3) * np_ * 4
    assert misc_used <= misc
    size = 1024 + ns * a_slot + nz * z_slot + 2 * ps * pbuf + nraw * raw_s + tables + misc
    assert m + misc_used + 1023 <= size <= k_smem
    assert ns >= 2 and nz >= 4
