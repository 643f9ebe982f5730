"""Accuracy metrics used to compare a GPU result with the oracle.

relative L2 ([aiter#7752] "Kernel": "Relative L2 against an fp32 reference"):
    ||y - r||_2 / ||r||_2 over all outputs, in float64.
error ratio ([aiter#7247] "Test Result": fraction of outputs outside tolerance
against a reference GEMM):
    mean( |y - r| > atol + rtol * |r| ).
bf16 ulp: the spacing of the bfloat16 grid at |r|, used to express
differences in units of the output format.

Parity: pinned in tests/test_oracle_gemm.py (the bf16 output-rounding floor
of relative L2 matches the 1.7e-3 of [aiter#7752]) and tests/test_oracle_metrics.py.
"""

import numpy as np


def rel_l2(y, r) -> float:
    y = np.asarray(y, dtype=np.float64)
    r = np.asarray(r, dtype=np.float64)
    den = np.linalg.norm(r.ravel())
    num = np.linalg.norm((y - r).ravel())
    if den == 0.0:
        return 0.0 if num == 0.0 else float("inf")
    return float(num / den)


def error_ratio(y, r, atol: float, rtol: float) -> float:
    y = np.asarray(y, dtype=np.float64)
    r = np.asarray(r, dtype=np.float64)
    if y.size == 0:
        return 0.0
    return float(np.mean(np.abs(y - r) > atol + rtol * np.abs(r)))


def bf16_ulp(r) -> np.ndarray:
    """Spacing of the bfloat16 grid at |r| (2^-133 below the normal range)."""
    r = np.abs(np.asarray(r, dtype=np.float64))
    _, ex = np.frexp(r)
    e = np.where(r == 0, -126, np.maximum(ex - 1, -126))
    return np.ldexp(1.0, e - 7)

