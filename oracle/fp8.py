"""Values of 8-bit floating-point codes, for the 8-bit paged cache.

Test infrastructure only (see ``oracle/__init__.py``).

The pages store the cache in bf16 and say nothing of 8-bit storage.  The
8-bit cache stores each element as an FP8 E4M3 code, the format of the Open
Compute Project's "OCP 8-bit Floating Point Specification (OFP8)": bit 7 is
the sign, bits 6-3 the exponent with bias 7, bits 2-0 the mantissa.  An
exponent field of 0 is subnormal (value m/8 * 2^-6); otherwise the value is
(1 + m/8) * 2^(e-7).  There is no infinity; S.1111.111 (0x7F, 0xFF) is NaN,
so the largest finite magnitude is 1.75 * 2^8 = 448.  An element of a pool
stands for scale * value(code) with one scale per pool.
"""
from __future__ import annotations

import numpy as np


def e4m3_value(codes) -> np.ndarray:
    """float64 value of each E4M3 code (uint8 array, or a torch uint8 tensor)."""
    if hasattr(codes, "numpy"):
        codes = codes.numpy()
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    mag = np.where((c & 0x7F) == 0x7F, np.nan, mag)
    return sign * mag


def dequantize(codes, scale: float) -> np.ndarray:
    """scale * value(code), in float64: the element a code stands for."""
    return float(scale) * e4m3_value(codes)


def e4m3_round(x) -> np.ndarray:
    """The E4M3 code nearest to each value (uint8): ties go to the even code, magnitudes above 448 saturate.

    x holds the values to encode, already in the precision in which they were
    formed (float32 for the 8-bit cache: x * (1/scale), both rounded to
    float32).  The sign bit follows the sign of x, so negative values that
    round to zero give -0 (0x80).  NaN is not encoded here.
    """
    x = np.asarray(x, dtype=np.float64)
    table = e4m3_value(np.arange(0x7F, dtype=np.uint8))          # the 127 non-negative finite values, increasing
    a = np.minimum(np.abs(x), table[-1])
    hi = np.searchsorted(table, a, side="left")                   # first value >= |x|
    hi = np.minimum(hi, len(table) - 1)
    lo = np.maximum(hi - 1, 0)
    d_lo, d_hi = a - table[lo], table[hi] - a
    take_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))     # equal distance: the even code
    code = np.where(take_hi, hi, lo).astype(np.uint8)
    code = np.where(a == table[hi], hi, code).astype(np.uint8)    # exact values
    return np.where(np.signbit(x), code | 0x80, code).astype(np.uint8)


def quantize(x, scale: float) -> np.ndarray:
    """Codes of the 8-bit cache for bf16/float32 values x: e4m3_round(float32(x) * float32(1 / float32(scale)))."""
    if hasattr(x, "float"):
        x = x.float().numpy()
    inv = np.float32(1.0) / np.float32(scale)
    return e4m3_round(np.asarray(x, dtype=np.float32) * inv)
