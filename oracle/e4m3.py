"""OCP 8-bit floating point E4M3 codec, written from the format definition.

TEST INFRASTRUCTURE ONLY (see package docstring).

E4M3 (the "fn" variant of the OCP 8-bit floating point specification): one sign
bit, four exponent bits with bias 7, three mantissa bits.
  * exponent field 0: subnormal, value = (-1)^s * 2^-6 * (m / 8)
  * exponent field 1..15: normal, value = (-1)^s * 2^(e - 7) * (1 + m / 8)
  * exponent 15 with mantissa 7 (S.1111.111) is NaN; there are no infinities.
The largest finite magnitude is 2^8 * 1.75 = 448; the smallest subnormal is
2^-9.

Encoding rounds to the nearest representable value, ties to the code with an
even mantissa (round-to-nearest-even), and saturates: magnitudes beyond 448
become +-448 ("satfinite").  NaN inputs encode to NaN.

The page this path comes from ("从理论到实现…" §4.1) quantises K with a
dynamic scale 127/amax, the int8 range; for the e4m3 format the matching
constant is the largest finite value, 448.
"""

from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


def _decode_one(code: int) -> float:
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * (2.0 ** -6) * (m / 8.0)
    return s * (2.0 ** (e - 7)) * (1.0 + m / 8.0)


_TABLE = np.array([_decode_one(c) for c in range(256)], dtype=np.float64)
# non-negative finite codes 0x00..0x7E are increasing in value
_POS_CODES = np.arange(0x7F, dtype=np.int64)
_POS_VALUES = _TABLE[:0x7F]


def e4m3_decode(codes) -> np.ndarray:
    """uint8 codes -> fp64 values (exact)."""
    return _TABLE[np.asarray(codes, dtype=np.uint8).astype(np.int64)]


def e4m3_encode_rne_satfinite(x) -> np.ndarray:
    """Values (any float dtype, taken exactly) -> uint8 e4m3 codes, RNE, satfinite."""
    x = np.asarray(x, dtype=np.float64)
    mag = np.abs(x)
    sat = np.minimum(mag, E4M3_MAX)
    # index of the largest representable value <= sat
    lo = np.searchsorted(_POS_VALUES, sat, side="right") - 1
    lo = np.clip(lo, 0, len(_POS_VALUES) - 1)
    hi = np.minimum(lo + 1, len(_POS_VALUES) - 1)
    v_lo = _POS_VALUES[lo]
    v_hi = _POS_VALUES[hi]
    d_lo = sat - v_lo
    d_hi = v_hi - sat
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi != lo) & ((_POS_CODES[hi] & 1) == 0))
    code = np.where(pick_hi, _POS_CODES[hi], _POS_CODES[lo]).astype(np.int64)
    code = np.where(np.signbit(x), code | 0x80, code)
    code = np.where(np.isnan(x), 0x7F, code)
    return code.astype(np.uint8)
