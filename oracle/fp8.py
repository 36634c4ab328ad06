"""e4m3 (fp8) decoding for the oracle (test infrastructure only).

The e4m3 byte format (the OCP 8-bit floating point "E4M3" encoding): bit 7 sign, bits 6..3
exponent with bias 7, bits 2..0 mantissa. Exponent field 0 is subnormal,
value = mantissa / 8 * 2^-6; otherwise value = (1 + mantissa / 8) * 2^(exponent - 7).
There are no infinities; exponent 15 with mantissa 7 (bytes 0x7F, 0xFF) is NaN, so the
largest finite magnitude is 1.75 * 2^8 = 448.
"""
from __future__ import annotations

import numpy as np


def decode_e4m3(codes) -> np.ndarray:
    """uint8 codes (any shape) -> float64 values (NaN for 0x7F / 0xFF)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag
