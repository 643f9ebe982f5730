"""Accuracy metrics used to compare a GPU result with the oracle.

relative L2 ([aiter#7752] "Kernel": "Relative L2 against an fp32 reference"):
    ||y - r||_2 / ||r||_2 over all outputs, in float64.
error ratio ([aiter#7247] "Test Result": fraction of outputs outside tolerance
against a reference GEMM):
    mean( |y - r| > atol + rtol * |r| ).
element-wise bound for a float32-accumulated result rounded once to bf16:
    |y - r| <= ulp_bf16(r) + c * 2^-24 * sum_k |a_k w_k| * |scales|
i.e. one bf16 rounding plus float32 summation error (derived from the
arithmetic: at most K additions of terms bounded by the absolute sum).

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


def within_fp32_accum_bf16_bound(y, r, abs_sum, n_terms: int, c: float = 2.0) -> np.ndarray:
    """Boolean mask: |y - r| <= ulp_bf16(r) + c * n_terms * 2^-24 * abs_sum.

    abs_sum is the sum of |terms| that make up r (same shape as r). The first
    term is one bf16 rounding of a value within the float32 error of r (a bf16
    ulp at the rounded value is at most one ulp at r, up to a binade edge, so
    one full ulp covers the half-ulp rounding plus the binade case); the second
    is the classic bound for recursive float32 summation of n_terms terms,
    with slack c for the product and scale roundings.
    """
    y = np.asarray(y, dtype=np.float64)
    r = np.asarray(r, dtype=np.float64)
    tol = bf16_ulp(r) + c * n_terms * 2.0 ** -24 * np.asarray(abs_sum, dtype=np.float64)
    return np.abs(y - r) <= tol
