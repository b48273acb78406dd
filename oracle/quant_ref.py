"""Per-token group quantiser of the latent cache, float32 semantics.

Test infrastructure only (see the package docstring).

QSVD paper notes, 实验关键数据 (W8A8 / W8A4 / W4A4 table) and QSVD digest,
Method, Step 3: the buffered latent C_qkv is quantised to 8 or 4 bits after
the H2 rotation.  The pages fix neither grid nor rounding; the readings taken
here (and in the CUDA library) are:

* symmetric grid [-qmax, qmax], qmax = 7 (int4) or 127 (int8);
* one scale per token and per group of ``group`` contiguous channels:
  amax = max |c| over the group (float32), s32 = amax / qmax (IEEE float32
  division, round to nearest even), s16 = float16(s32) (round to nearest
  even; saturated at 65504 with an overflow flag);
* code = 0 if s16 == 0, else clamp(rint(c / float(s16)), -qmax, qmax) with
  float32 division and round-half-to-even;
* int4 packing: element 2j in the low nibble, 2j+1 in the high nibble, both
  in two's complement.

Dequantised value: float(code) * float(s16), exact in float32.
"""
from __future__ import annotations

import numpy as np

QMAX = {4: 7, 8: 127}
F16_MAX = np.float32(65504.0)


def quantize(c32: np.ndarray, bits: int, group: int):
    """Quantise the last axis of ``c32`` (float32 values) in groups.

    Returns (codes int8 (..., r), scales float16 (..., r/group),
    overflow bool (..., r/group))."""
    c = np.asarray(c32, dtype=np.float32)
    r = c.shape[-1]
    if r % group:
        raise ValueError("group must divide r")
    qmax = np.float32(QMAX[bits])
    g = c.reshape(c.shape[:-1] + (r // group, group))
    amax = np.max(np.abs(g), axis=-1)
    s32 = (amax / qmax).astype(np.float32)
    overflow = s32 > F16_MAX
    s32 = np.minimum(s32, F16_MAX)
    s16 = s32.astype(np.float16)
    sf = s16.astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = (g / sf[..., None]).astype(np.float32)
    codes = np.rint(ratio)
    codes = np.where(sf[..., None] == 0, np.float32(0), codes)
    codes = np.clip(codes, -qmax, qmax).astype(np.int8)
    return codes.reshape(c.shape), s16, overflow


def dequantize(codes: np.ndarray, scales: np.ndarray, group: int) -> np.ndarray:
    """float(code) * float(scale) per group (exact in float32)."""
    codes = np.asarray(codes, np.int8)
    r = codes.shape[-1]
    g = codes.reshape(codes.shape[:-1] + (r // group, group)).astype(np.float32)
    out = g * np.asarray(scales, np.float16).astype(np.float32)[..., None]
    return out.reshape(codes.shape)


def pack_int4(codes: np.ndarray) -> np.ndarray:
    """Two int4 codes per byte: element 2j low nibble, 2j+1 high nibble."""
    c = np.asarray(codes, np.int8).astype(np.int16)
    lo = c[..., 0::2] & 0xF
    hi = c[..., 1::2] & 0xF
    return (lo | (hi << 4)).astype(np.uint8)


def unpack_int4(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, np.uint8).astype(np.int16)
    lo = p & 0xF
    hi = (p >> 4) & 0xF
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), np.int8)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out
