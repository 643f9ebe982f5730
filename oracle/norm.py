"""Fused residual add + RMSNorm + per-token-group activation quantisation -- the step
upstream of the a8w8 GEMM (``add_rmsnorm_quant`` in the decode-window kernel table of
[mi210 docs/43] "43-ck-int8-gemm-gfx90a.md", Rounds 40-41). TEST INFRASTRUCTURE ONLY.

The pages name the kernel but print no formula. Reading (the plainest one consistent
with a residual stream kept in bf16 feeding the 1x128 activation quantiser):

    h[m,k]   = bf16( float32(x[m,k]) + float32(residual[m,k]) )    new residual stream
    r[m]     = 1 / sqrt( (1/K) sum_k h[m,k]^2 + eps )
    y[m,k]   = h[m,k] * r[m] * gamma[k]
    (q, a_scale) = quant_act_per_token_group(float32(y))            1x128 groups, amax/448

The residual add is an fp32 add of two bf16 values rounded once to bf16 (as the GPU
does it); the mean square, r and y are float64 here and y is rounded to float32 before
quantisation, the precision in which the kernel takes the quantisation decision (its own
mean square and r are float32, so a code may differ from this one by one step where
y / a_scale lies within float32 error of a rounding midpoint -- the parity test checks
the codes exactly elsewhere and the neighbouring code there).

Parity: pinned in tests/test_oracle_norm.py (residual add against torch's bf16 cast; the
norm against torch's float64 rms_norm; closed forms on constant rows; the zero row;
planted mistakes).
"""

import numpy as np

from .bf16 import round_to_bf16
from .quant import quant_act_per_token_group


def add_residual(x, residual) -> np.ndarray:
    """h = bf16(float32(x) + float32(residual)), as float64 holding bf16 values."""
    s = (np.asarray(x, dtype=np.float32) + np.asarray(residual, dtype=np.float32)).astype(np.float64)
    return round_to_bf16(s)


def rmsnorm(h, gamma, eps: float) -> np.ndarray:
    """y = h / sqrt(mean(h^2) + eps) * gamma, float64, row by row."""
    h = np.asarray(h, dtype=np.float64)
    g = np.asarray(gamma, dtype=np.float64)
    ms = np.mean(h * h, axis=1, keepdims=True)
    r = 1.0 / np.sqrt(ms + eps)
    return h * r * g[None, :]


def add_rmsnorm_quant(x, residual, gamma, eps: float):
    """Returns (h [M,K] float64 of bf16 values, y [M,K] float64, q [M,K] uint8 codes,
    a_scale [M,K/128] float32)."""
    h = add_residual(x, residual)
    y = rmsnorm(h, gamma, eps)
    q, a_s = quant_act_per_token_group(y.astype(np.float32))
    return h, y, q, a_s
