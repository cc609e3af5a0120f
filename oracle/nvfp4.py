"""Exact NVFP4 decode: e2m1 element codes times one e4m3 scale per 16 consecutive elements.

TEST INFRASTRUCTURE (see the package docstring).

The pages only say that the simulated results use FP4 KV (paper summary, fdeinterviews.com,
roofline paragraph: "in FP4"). The storage format used here is NVFP4 as the workload defines it:
e2m1 values, one fp8-e4m3 scale per 16 contiguous elements along the head dimension, no second-level
tensor scale. Element 2i of a row sits in the LOW nibble of byte i, element 2i+1 in the high nibble.

Both decoders are written from the public bit-level definitions:
* FP4 E2M1 (OCP Microscaling Formats v1.0): 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit;
  exponent field 0 is subnormal (value = mantissa * 0.5); no inf or NaN. Magnitudes
  {0, 0.5, 1, 1.5, 2, 3, 4, 6}.
* FP8 E4M3 (OCP 8-bit floating point, the "fn" variant): 1 sign, 4 exponent bits (bias 7), 3 mantissa
  bits; exponent field 0 is subnormal (mantissa/8 * 2^-6); S.1111.111 is NaN; no inf; max 448.
"""

from __future__ import annotations

import math

import numpy as np


def e2m1_value(code: int) -> float:
    """Value of a 4-bit E2M1 code."""
    code = int(code) & 0xF
    sign = -1.0 if code & 0x8 else 1.0
    e = (code >> 1) & 0x3
    m = code & 0x1
    if e == 0:
        mag = 0.5 * m
    else:
        mag = math.ldexp(1.0 + 0.5 * m, e - 1)
    return sign * mag


def e4m3_value(byte: int) -> float:
    """Value of an 8-bit E4M3 ("fn") code."""
    byte = int(byte) & 0xFF
    sign = -1.0 if byte & 0x80 else 1.0
    e = (byte >> 3) & 0xF
    m = byte & 0x7
    if e == 0xF and m == 0x7:
        return math.nan
    if e == 0:
        mag = math.ldexp(m / 8.0, -6)
    else:
        mag = math.ldexp(1.0 + m / 8.0, e - 7)
    return sign * mag


_E2M1 = np.array([e2m1_value(c) for c in range(16)], dtype=np.float64)
_E4M3 = np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)


def nvfp4_dequant(codes, scales) -> np.ndarray:
    """Decode packed NVFP4 rows to fp64.

    codes  uint8 [..., d/2]  (element 2i in the low nibble of byte i, 2i+1 in the high nibble)
    scales uint8 [..., d/16] (E4M3 bytes; scale j applies to elements 16j .. 16j+15)
    returns fp64 [..., d]; every value is exactly code_value * scale_value.
    """
    codes = np.asarray(codes.cpu().numpy() if hasattr(codes, "cpu") else codes, dtype=np.uint8)
    scales = np.asarray(scales.cpu().numpy() if hasattr(scales, "cpu") else scales, dtype=np.uint8)
    lo = _E2M1[codes & 0xF]
    hi = _E2M1[codes >> 4]
    elems = np.stack([lo, hi], axis=-1).reshape(*codes.shape[:-1], codes.shape[-1] * 2)
    d = elems.shape[-1]
    sc = np.repeat(_E4M3[scales], 16, axis=-1)
    assert sc.shape[-1] == d, "one scale per 16 elements"
    return elems * sc


# ------------------------------------------------------------------------------------------------
# Encoding (the quantiser of the append path). The pages give no rule beyond "FP4"; the workload
# definition fixes the scale as the block absmax / 6 in E4M3. Every rounding decision is taken in
# fp32, the precision a device quantiser computes in, and each step follows the format definitions:
#   1. amax = max |x| over the 16-element block                       (exact)
#   2. r = fp32(amax / 6)                                             (IEEE fp32 division, nearest)
#   3. scale = the E4M3 value nearest to r, ties to the even code;
#      r above the largest finite value 448 gives 448 ("satfinite")
#   4. y_i = fp32(x_i / scale), or y_i = x_i when the scale is 0     (IEEE fp32 division)
#   5. code_i = the E2M1 value nearest to y_i, ties to the even code, |y| > 6 gives 6; the sign bit
#      is set only for a non-zero magnitude (a value that rounds to zero is stored as +0)
# ------------------------------------------------------------------------------------------------

_E2M1_MAG = _E2M1[:8]  # magnitudes of codes 0..7
_E4M3_FINITE = _E4M3[:0x7F]  # non-negative finite E4M3 values, codes 0x00..0x7E


def _nearest_even(a, table):
    """Index of the entry of ``table`` (ascending) nearest to each a (fp64, exact inputs); ties go
    to the even index, which is the even code for both formats."""
    a = np.asarray(a, dtype=np.float64)
    d = np.abs(a[..., None] - table)
    dmin = d.min(axis=-1, keepdims=True)
    tie = d == dmin
    idx = np.arange(table.shape[0])
    # among the (at most two, adjacent) nearest entries prefer the even index
    even_pick = np.where(tie & (idx % 2 == 0), idx, table.shape[0] + 1).min(axis=-1)
    any_pick = np.where(tie, idx, table.shape[0] + 1).min(axis=-1)
    return np.where(even_pick <= table.shape[0], even_pick, any_pick)


def e4m3_encode_satfinite(r) -> np.ndarray:
    """E4M3 code (uint8) of non-negative fp32 values: nearest, ties to even, clamped to 448."""
    r = np.asarray(r, dtype=np.float32).astype(np.float64)
    code = _nearest_even(np.minimum(r, 448.0), _E4M3_FINITE)
    return code.astype(np.uint8)


def e2m1_encode_satfinite(y) -> np.ndarray:
    """E2M1 code (0..15) of fp32 values: nearest magnitude, ties to even, |y| > 6 gives 6, and
    the sign bit only on a non-zero magnitude."""
    y = np.asarray(y, dtype=np.float32).astype(np.float64)
    mag = _nearest_even(np.minimum(np.abs(y), 6.0), _E2M1_MAG).astype(np.uint8)
    sign = ((y < 0) & (mag > 0)).astype(np.uint8)
    return (mag | (sign << 3)).astype(np.uint8)


def nvfp4_encode(x):
    """Encode rows [..., d] (d a multiple of 16; any real dtype, taken as fp32) to NVFP4:
    returns (codes uint8 [..., d/2] with element 2i in the low nibble of byte i,
    scales uint8 [..., d/16] E4M3), following steps 1-5 above."""
    x = np.asarray(x.cpu().numpy() if hasattr(x, "cpu") else x).astype(np.float32)
    *lead, d = x.shape
    assert d % 16 == 0
    xb = x.reshape(*lead, d // 16, 16)
    amax = np.abs(xb).max(axis=-1)
    r = (amax / np.float32(6.0)).astype(np.float32)
    s_code = e4m3_encode_satfinite(r)
    sd = _E4M3[s_code].astype(np.float32)
    safe = np.where(sd > 0, sd, np.float32(1.0)).astype(np.float32)
    y = (xb / safe[..., None]).astype(np.float32)
    codes = e2m1_encode_satfinite(y).reshape(*lead, d // 2, 2)
    packed = (codes[..., 0] | (codes[..., 1] << 4)).astype(np.uint8)
    return packed, s_code.reshape(*lead, d // 16)
