"""Every tiled TMA load's innermost coordinate starts on a 16-byte boundary.

A tiled bulk-tensor copy whose innermost coordinate times the element size
is not a multiple of 16 bytes is an illegal instruction on sm_100 (nothing
checks it before the copy runs).  This test reads the library's sources,
extracts the innermost coordinate of every `tma_load_*` call and of the two
inline-assembly loads (the tensor-core GEMV and the absorption), and
requires each to be one of the expressions below, each with the reason it
is aligned.  A new call site with a new expression fails here until it is
reviewed and added.
"""
import glob
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "rank_joint_qkv_b200", "csrc")

# expression -> why it is a multiple of 16 bytes
ALIGNED = {
    "0": "the box starts at the row's first element",
    # 16-bit maps: multiples of 64 elements (128 bytes)
    "64 * ki": "64 fp16/bf16 elements per K box",
    "64 * u": "64 fp16/bf16 elements per channel box",
    "64 * kb": "64 fp16/bf16 elements per channel box",
    "64": "the second 64-element box of a 128-wide row",
    "col": "h * 128 (prefill attention: d_h = 128)",
    "col + 64": "h * 128 + 64",
    "ch0 + 64 * lane": "the cluster rank times its channel width, a multiple of 64",
    "col0": "the GEMV's column tile, blockIdx.x * 64",
    "h * d_h + 64 * c": "the tensor-core absorption runs only for d_h % 64 == 0",
    # 8-bit maps (int8 / int4 codes, int8 query parts): multiples of 16 bytes
    "128 * u": "128 bytes per 128-channel int8 group",
    "ua * 64": "64 bytes per 128-channel int4 group",
    "(u >> 1) * (QB * 16)": "QB * 16 = 64 (int4) or 128 (int8) bytes per 128 channels",
}


def _args(s, i):
    """Arguments of the call whose '(' is at s[i], split at depth one."""
    depth, cur, out = 0, "", []
    for c in s[i:]:
        if c == "(":
            depth += 1
            if depth == 1:
                continue
        elif c == ")":
            depth -= 1
            if depth == 0:
                out.append(cur.strip())
                return out
        elif c == "," and depth == 1:
            out.append(cur.strip())
            cur = ""
            continue
        cur += c
    raise AssertionError("unbalanced call")


def _norm(e):
    return " ".join(e.split())


def test_every_tma_load_starts_on_a_16_byte_boundary():
    seen = []
    call = re.compile(r"\btma_load_\dd(?:_hint)?\(")
    for f in sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))):
        s = open(f).read()
        for m in call.finditer(s):
            line = s[s.rfind("\n", 0, m.start()) + 1:s.find("\n", m.start())]
            if "__device__" in line:          # the helper's own definition
                continue
            x = _norm(_args(s, m.end() - 1)[2])
            assert x in ALIGNED, f"{os.path.basename(f)}: unreviewed TMA x coordinate {x!r}"
            seen.append(x)
        # inline-assembly tiled loads outside the helpers: the coordinate is
        # the first "r" operand after the tensor map's "l" operand
        if os.path.basename(f) == "tc_common.cuh":
            continue
        for m in re.finditer(r'cp\.async\.bulk\.tensor\.\dd\.shared::cluster\.global', s):
            tail = s[m.end():m.end() + 600]
            mm = re.search(r'"l"\(reinterpret_cast<uint64_t>\(&\w+\)\),\s*"r"\(([^)]*)\)', tail)
            assert mm, f"{os.path.basename(f)}: tiled load without a recognisable coordinate"
            x = _norm(mm.group(1))
            assert x in ALIGNED, f"{os.path.basename(f)}: unreviewed TMA x coordinate {x!r}"
            seen.append(x)
    assert len(seen) >= 25            # every path's loads were found
    assert "col0" in seen and "h * d_h + 64 * c" in seen
