"""MX32 variant of the a8w8 GEMM: power-of-two (E8M0) scales on 32-wide K groups, with
32x32 weight blocks -- ``gemm_a8w8_blockscale_mxscale`` / its batched form in
[aiter#7247] (ROCm/aiter PR #7247, "Motivation": "MX32 (w_scale_block 32x32)";
"Technical Details": MX32 dense shapes and batched b=8, N=1024, K=4096). TEST
INFRASTRUCTURE ONLY.

The page gives the block shape and the name only. Readings (the plainest ones the rest
supports; listed in the design notes):
  * "mxscale" is the OCP microscaling scale: an 8-bit biased exponent (E8M0), value
    2^(code - 127); code 255 (NaN) is never produced.
  * Activations are quantised per token per 1x32 K group (the MX block along K), weights
    per 32x32 block, both to OCP e4m3fn.
  * The exponent is the smallest one that keeps the group within the e4m3 range, the
    power-of-two counterpart of the 128-block rule scale = amax / 448:
        r = float32(amax) / float32(448)                 (one IEEE float32 division)
        e = ceil(log2 r), read exactly from r's bits (exponent, +1 if any mantissa bit)
        code = clamp(e + 127, 0, 254);  amax == 0 gives code 0
    so amax / 2^e lies in (224, 448] and nothing saturates except where the division's
    rounding lands exactly on a power of two.
  * codes = e4m3_rn_sat(x * 2^-e) (exact power-of-two scaling, one RN-sat rounding).
  * out[m,n] = sum_g 2^(ea[m,g] + ew[n//32, g]) * sum_{k in g} A[m,k] W[n,k], float64
    here (exact per group), rounded once to bf16.
  * W is K-major [N, K] like the 128-block path (the pages' "bpreshuffle" is an AMD
    register layout, not part of what is computed).

Parity: pinned in tests/test_oracle_mx.py (E8M0 decode exhaustive; the exponent rule on
exact powers of two and their neighbours; the (224, 448] property; a scalar restatement
with ml_dtypes' encoder; exact rational brute force; reduction to the 128-block oracle
when the scales are constant over 128-wide groups and 128-row blocks; planted mistakes).
"""

import numpy as np

from .bf16 import round_to_bf16
from .e4m3 import decode, encode_rn_sat

GROUP = 32
E8M0_BIAS = 127


def e8m0_decode(code) -> np.ndarray:
    """2^(code - 127) as float64 (code 255, NaN in the format, is rejected)."""
    c = np.asarray(code, dtype=np.int64)
    assert np.all((c >= 0) & (c <= 254)), "E8M0 code 255 (NaN) or out of range"
    return np.ldexp(1.0, c - E8M0_BIAS)


def exponent_for_amax(amax) -> np.ndarray:
    """E8M0 code of the smallest power of two 2^e with amax / 2^e <= 448 (float32 rule)."""
    a = np.asarray(amax, dtype=np.float32)
    r = (a / np.float32(448.0)).astype(np.float32)
    bits = r.view(np.uint32).astype(np.int64)
    ex = (bits >> 23) & 0xFF
    man = bits & 0x7FFFFF
    e_norm = ex - 127 + (man != 0)
    # subnormal r (amax below 448 * 2^-126): ceil(log2 r) from the mantissa's top bit
    top = np.floor(np.log2(np.maximum(man, 1))).astype(np.int64)  # index of the leading mantissa bit
    e_sub = -149 + top + ((man & ((np.int64(1) << top) - 1)) != 0)
    e = np.where(ex == 0, e_sub, e_norm)
    code = np.clip(e + E8M0_BIAS, 0, 254)
    return np.where(a == 0, 0, code).astype(np.uint8)


def _scale_codes(blk_amax):
    return exponent_for_amax(blk_amax)


def quant_act_mx32(x):
    """x: [M, K] float32 (bf16 values). Returns (codes uint8 [M, K], e8m0 uint8 [M, K/32])."""
    x = np.asarray(x, dtype=np.float32)
    M, K = x.shape
    assert K % GROUP == 0
    G = K // GROUP
    codes = np.empty((M, K), dtype=np.uint8)
    ex = np.empty((M, G), dtype=np.uint8)
    for g in range(G):
        blk = x[:, g * GROUP:(g + 1) * GROUP]
        c = _scale_codes(np.max(np.abs(blk), axis=1))
        ex[:, g] = c
        inv = np.ldexp(np.float32(1.0), -(c.astype(np.int64) - E8M0_BIAS)).astype(np.float32)  # exact 2^-e
        codes[:, g * GROUP:(g + 1) * GROUP] = encode_rn_sat((blk.astype(np.float64) * inv[:, None]).astype(np.float32))
    return codes, ex


def quant_weight_mx32(w):
    """w: [N, K] float32. Returns (codes uint8 [N, K], e8m0 uint8 [ceil(N/32), K/32]); a
    partial last block of rows is quantised over the rows it has."""
    w = np.asarray(w, dtype=np.float32)
    N, K = w.shape
    assert K % GROUP == 0
    NB, G = (N + GROUP - 1) // GROUP, K // GROUP
    codes = np.empty((N, K), dtype=np.uint8)
    ex = np.empty((NB, G), dtype=np.uint8)
    for nb in range(NB):
        r0, r1 = nb * GROUP, min(N, (nb + 1) * GROUP)
        for g in range(G):
            blk = w[r0:r1, g * GROUP:(g + 1) * GROUP]
            c = _scale_codes(np.max(np.abs(blk)))
            ex[nb, g] = c
            inv = np.ldexp(1.0, -(int(c) - E8M0_BIAS))
            codes[r0:r1, g * GROUP:(g + 1) * GROUP] = encode_rn_sat((blk.astype(np.float64) * inv).astype(np.float32))
    return codes, ex


def gemm_a8w8_mx32_ref(A_q, a_e, W_q, w_e) -> np.ndarray:
    """Unrounded float64 result [M, N] of the MX32 block-scaled GEMM."""
    A = decode(A_q)
    W = decode(W_q)
    M, K = A.shape
    N = W.shape[0]
    assert W.shape[1] == K and K % GROUP == 0
    G = K // GROUP
    sa = e8m0_decode(a_e)
    sw = e8m0_decode(w_e)
    assert sa.shape == (M, G) and sw.shape == ((N + GROUP - 1) // GROUP, G)
    nb_of_n = np.arange(N) // GROUP
    out = np.zeros((M, N), dtype=np.float64)
    for g in range(G):
        ks = slice(g * GROUP, (g + 1) * GROUP)
        out += (sa[:, g][:, None] * sw[nb_of_n, g][None, :]) * (A[:, ks] @ W[:, ks].T)
    return out


def gemm_a8w8_mx32(A_q, a_e, W_q, w_e):
    """Returns (ref float64 [M, N], out float64 [M, N] holding bf16 values)."""
    ref = gemm_a8w8_mx32_ref(A_q, a_e, W_q, w_e)
    return ref, round_to_bf16(ref)


def batched_gemm_a8w8_mx32(A_q, a_e, W_q, w_e):
    """b independent MX32 GEMMs: A_q [b, M, K], a_e [b, M, K/32], W_q [b, N, K],
    w_e [b, N/32, K/32]. Returns (ref [b, M, N], out [b, M, N])."""
    refs = [gemm_a8w8_mx32_ref(A_q[i], a_e[i], W_q[i], w_e[i]) for i in range(len(A_q))]
    ref = np.stack(refs)
    return ref, round_to_bf16(ref)
