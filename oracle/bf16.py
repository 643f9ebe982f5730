"""bfloat16 rounding (round to nearest, ties to even) from float64.

bfloat16 = float32 with the low 16 bits dropped: 1 sign, 8 exponent (bias 127),
7 stored mantissa bits, i.e. 8 significant bits. For |v| >= 2^-126 the spacing
of the grid at v is 2^(floor(log2|v|) - 7); below that (subnormals) it is
2^-133. Rounding is done in one step from the float64 value, so there is no
double rounding through float32. Overflow (a result above the largest finite
bf16, (2 - 2^-7) * 2^127) gives +-inf.

Parity: pinned in tests/test_oracle_bf16.py (against torch's float32->bf16 cast
on float32-representable values, and against exact rational rounding with
Python's fractions on values that are not float32-representable).
"""

import numpy as np

BF16_MAX = (2.0 - 2.0 ** -7) * 2.0 ** 127


def round_to_bf16(v) -> np.ndarray:
    """float64 array -> float64 array holding the RN-even bfloat16 values."""
    v = np.asarray(v, dtype=np.float64)
    out = np.zeros_like(v)
    nz = np.isfinite(v) & (v != 0.0)
    vv = v[nz]
    _, ex = np.frexp(vv)  # |vv| = m * 2^ex with m in [0.5, 1)
    exp_floor = np.maximum(ex - 1, -126)
    q = np.ldexp(1.0, exp_floor - 7)
    r = np.rint(vv / q) * q  # vv / q is exact: power-of-two scaling
    r = np.where(np.abs(r) > BF16_MAX, np.copysign(np.inf, r), r)
    out[nz] = r
    out[~nz] = v[~nz]  # zeros (with sign), inf and nan pass through
    return out


def to_bits(v_bf16_values) -> np.ndarray:
    """Exact bfloat16 values (float64) -> uint16 bit patterns."""
    f = np.asarray(v_bf16_values, dtype=np.float64).astype(np.float32)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


def from_bits(bits) -> np.ndarray:
    """uint16 bfloat16 bit patterns -> float64 values (exact)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)
