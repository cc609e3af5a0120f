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
