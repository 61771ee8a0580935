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
