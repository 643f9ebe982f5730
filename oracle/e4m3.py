"""OCP FP8 E4M3 ("e4m3fn") codec, written from the format definition.

Format: bit 7 sign, bits 6..3 biased exponent (bias 7), bits 2..0 mantissa.
  exponent field 0          -> subnormal, value = (-1)^s * m * 2^-9
  exponent field 1..15      -> normal,    value = (-1)^s * (1 + m/8) * 2^(e-7)
  exponent 15, mantissa 7   -> NaN (the only non-finite code; no infinities)
Largest finite magnitude: 1.75 * 2^8 = 448. Smallest subnormal: 2^-9.

The a8w8 block-scale quantisers of the pages store e4m3 codes with a
round-to-nearest-even, saturate-to-finite conversion ("RN-sat"): magnitudes at
or above 448 become 448, everything else rounds to the nearest grid point with
ties to the even code. NaN inputs are out of scope (inputs are finite).

Parity: pinned in tests/test_oracle_e4m3.py (exhaustive decode against two
independent libraries, hand values from the definition, every midpoint, and
random values against library casts inside the finite range).
"""

import numpy as np

E4M3_MAX = 448.0


def decode_code(c: int) -> float:
    """Value of one e4m3 code, straight from the bit fields."""
    c = int(c) & 0xFF
    sign = -1.0 if (c & 0x80) else 1.0
    e = (c >> 3) & 0xF
    m = c & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return sign * m * 2.0 ** -9
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


DECODE_TABLE = np.array([decode_code(c) for c in range(256)], dtype=np.float64)

# Non-negative finite grid: codes 0x00..0x7E in code order, strictly increasing.
_POS_GRID = DECODE_TABLE[:0x7F].copy()


def decode(codes) -> np.ndarray:
    """uint8 codes (any shape) -> float64 values."""
    return DECODE_TABLE[np.asarray(codes, dtype=np.uint8)]


def encode_rn_sat(v) -> np.ndarray:
    """Finite values (float32/float64, any shape) -> e4m3 codes, RN-even, saturating.

    The sign bit of the code is the sign bit of the input, so -0.0 and small
    negative values that round to zero give 0x80.
    """
    v = np.asarray(v, dtype=np.float64)
    neg = np.signbit(v)
    a = np.minimum(np.abs(v), E4M3_MAX)
    hi = np.searchsorted(_POS_GRID, a, side="left")  # grid[hi-1] < a <= grid[hi]
    hi = np.clip(hi, 0, 0x7E)
    lo = np.maximum(hi - 1, 0)
    d_lo = a - _POS_GRID[lo]
    d_hi = _POS_GRID[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(a == _POS_GRID[hi], hi, np.where(pick_hi, hi, lo)).astype(np.uint8)
    return np.where(neg, code | 0x80, code).astype(np.uint8)
