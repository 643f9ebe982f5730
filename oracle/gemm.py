"""The a8w8 block-scaled GEMM and the companion bf16 GEMM, in float64.

a8w8 block scale (the operation behind ``gemm_a8w8_blockscale`` in
[cookbook#8] and [aiter#7752] "Kernel"): with A codes [M, K] and their
per-token-group scales a_s [M, G], W codes [N, K] and their 128x128 block
scales w_s [ceil(N/128), G], G = K/128,

    out[m, n] = sum_g  a_s[m, g] * w_s[n // 128, g] * P_g[m, n]
    P_g[m, n] = sum_{k in group g} decode(A[m, k]) * decode(W[n, k])

The reported output is that sum rounded once to bfloat16 (RN-even). The GPU
accumulates in float32; the oracle keeps float64, in which every P_g is exact
(products of two e4m3 values have at most 8 significant bits and lie in
[2^-18, 2^18); a sum of 128 of them spans fewer than 53 bits).

bf16 GEMM (the small-N router / indexer companion, ``tgemm`` in
[cookbook#8] and the BF16 rows of [aiter#7247]): out = A @ W^T with A [M, K]
and W [N, K] bf16, summed in float64, rounded once to bf16 or to float32.

A library matmul (numpy float64) serves as the inner-product step, as the
definition allows; nothing is blocked, fused or reordered beyond the sum over
groups the definition itself states.

Parity: pinned in tests/test_oracle_gemm.py (exact rational brute force on tiny
shapes, integer-valued exact cases, scale linearity, the all-ones-scale
reduction to a plain matmul, the bf16 output-rounding floor of [aiter#7752],
and plant-a-mistake checks).
"""

import numpy as np

from .e4m3 import decode
from .bf16 import round_to_bf16

GROUP = 128


def gemm_a8w8_blockscale_ref(A_q, a_s, W_q, w_s) -> np.ndarray:
    """Unrounded float64 result [M, N]."""
    A = decode(A_q)
    W = decode(W_q)
    a_s = np.asarray(a_s, dtype=np.float32).astype(np.float64)
    w_s = np.asarray(w_s, dtype=np.float32).astype(np.float64)
    M, K = A.shape
    N, K2 = W.shape
    assert K == K2 and K % GROUP == 0
    G = K // GROUP
    assert a_s.shape == (M, G)
    assert w_s.shape == ((N + 127) // 128, G)
    nb_of_n = np.arange(N) // 128
    out = np.zeros((M, N), dtype=np.float64)
    for g in range(G):
        ks = slice(g * GROUP, (g + 1) * GROUP)
        P = A[:, ks] @ W[:, ks].T
        out += (a_s[:, g][:, None] * w_s[nb_of_n, g][None, :]) * P
    return out


def gemm_a8w8_blockscale(A_q, a_s, W_q, w_s):
    """Returns (ref float64 [M, N], out float64 [M, N] holding bf16 values)."""
    ref = gemm_a8w8_blockscale_ref(A_q, a_s, W_q, w_s)
    return ref, round_to_bf16(ref)


def gemm_bf16_ref(A, W) -> np.ndarray:
    """A [M, K], W [N, K] (float arrays holding bf16 values) -> float64 [M, N]."""
    A = np.asarray(A, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    return A @ W.T


def gemm_bf16(A, W, out_fp32: bool = False):
    """Returns (ref float64, out): out rounded once to bf16, or to float32 if out_fp32."""
    ref = gemm_bf16_ref(A, W)
    out = ref.astype(np.float32).astype(np.float64) if out_fp32 else round_to_bf16(ref)
    return ref, out
