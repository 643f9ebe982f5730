"""Pins for the oracle's MX32 quantisers and GEMM (CPU only)."""

from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest

from oracle import e4m3, gemm as ogemm, mx
from fp8_block_scaled_a8w8_b200 import inputs


def test_e8m0_decode_exhaustive():
    codes = np.arange(255)
    np.testing.assert_array_equal(mx.e8m0_decode(codes), [2.0 ** (c - 127) for c in codes])
    with pytest.raises(AssertionError):
        mx.e8m0_decode(np.array([255]))


def test_exponent_rule_at_powers_of_two_and_neighbours():
    for k in range(-20, 20):
        exact = np.float32(448.0 * 2.0 ** k)
        assert mx.exponent_for_amax(exact) == 127 + k          # no rounding up at an exact fit
        above = np.nextafter(exact, np.float32(np.inf))
        assert mx.exponent_for_amax(above) == 127 + k + 1      # the next power of two
        below = np.nextafter(exact, np.float32(0))
        assert mx.exponent_for_amax(below) == 127 + k
    assert mx.exponent_for_amax(np.float32(0)) == 0
    assert mx.exponent_for_amax(np.float32(1e38)) == 127 + 118  # 2^117 < 1e38 / 448 < 2^118
    # subnormal ratio: amax = 448 * 2^-140 -> r = 2^-140 exactly
    assert mx.exponent_for_amax(np.float32(448.0 * 2.0 ** -140)) == 0  # clamped at code 0 (2^-127)


def test_scaled_group_max_lies_in_224_448():
    x = inputs.activation_bf16(64, 1024, 3, outliers=True).float().numpy()
    q, ex = mx.quant_act_mx32(x)
    for g in range(1024 // 32):
        amax = np.max(np.abs(x[:, g * 32:(g + 1) * 32]), axis=1).astype(np.float64)
        t = amax / mx.e8m0_decode(ex[:, g])
        assert np.all((t > 224) & (t <= 448))


def test_quant_scalar_restatement_with_ml_dtypes():
    x = inputs.activation_bf16(5, 256, 7).float().numpy()
    q, ex = mx.quant_act_mx32(x)
    for m in range(5):
        for g in range(256 // 32):
            blk = x[m, g * 32:(g + 1) * 32].astype(np.float64)
            amax = np.max(np.abs(blk))
            r = np.float32(np.float32(amax) / np.float32(448.0))
            e = int(np.ceil(np.log2(float(r))))  # r is normal here
            assert ex[m, g] == e + 127
            want = (blk / 2.0 ** e).astype(np.float32).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
            np.testing.assert_array_equal(q[m, g * 32:(g + 1) * 32], want)


def test_weight_blocks_and_partial_rows():
    w = inputs.weight_f32(70, 96, 11).numpy()  # 3 row blocks (last has 6 rows), 3 K groups
    q, ex = mx.quant_weight_mx32(w)
    assert ex.shape == (3, 3)
    for nb in range(3):
        for g in range(3):
            blk = w[nb * 32:min(70, nb * 32 + 32), g * 32:(g + 1) * 32]
            assert ex[nb, g] == mx.exponent_for_amax(np.max(np.abs(blk)))
            deq = e4m3.decode(q[nb * 32:min(70, nb * 32 + 32), g * 32:(g + 1) * 32]) * mx.e8m0_decode(ex[nb, g])
            assert np.all(np.abs(deq - blk) <= np.abs(blk) * 2.0 ** -4 + 2.0 ** -9 * mx.e8m0_decode(ex[nb, g]))


def _raw(M, N, K, seed):
    rng = np.random.default_rng(seed)
    A = inputs.random_e4m3_codes((M, K), seed)
    W = inputs.random_e4m3_codes((N, K), seed + 1)
    ae = rng.integers(110, 140, (M, K // 32)).astype(np.uint8)
    we = rng.integers(110, 140, ((N + 31) // 32, K // 32)).astype(np.uint8)
    return A, ae, W, we


def test_gemm_exact_rational_brute_force():
    A, ae, W, we = _raw(2, 40, 64, 5)
    ref = mx.gemm_a8w8_mx32_ref(A, ae, W, we)
    dA = [[Fraction(float(v)) for v in row] for row in e4m3.decode(A)]
    dW = [[Fraction(float(v)) for v in row] for row in e4m3.decode(W)]
    for m in range(2):
        for n in range(40):
            s, mag = Fraction(0), Fraction(0)
            for k in range(64):
                g = k // 32
                t = dA[m][k] * dW[n][k] * Fraction(2) ** (int(ae[m, g]) - 127) * Fraction(2) ** (int(we[n // 32, g]) - 127)
                s += t
                mag += abs(t)
            # each group's sum is exact in float64; only the sum over the 2 groups rounds
            assert abs(Fraction(ref[m, n]) - s) <= mag * Fraction(1, 2 ** 52)


def test_gemm_reduces_to_the_128_block_oracle():
    # scales constant over each 128-wide K group and 128-row weight block: the MX32 GEMM is
    # the 128-block GEMM with scales 2^e
    M, N, K = 5, 256, 384
    A, _, W, _ = _raw(M, N, K, 9)
    rng = np.random.default_rng(1)
    ae128 = rng.integers(115, 135, (M, K // 128)).astype(np.uint8)
    we128 = rng.integers(115, 135, (N // 128, K // 128)).astype(np.uint8)
    ae = np.repeat(ae128, 4, axis=1)
    we = np.repeat(np.repeat(we128, 4, axis=0), 4, axis=1)
    ref = mx.gemm_a8w8_mx32_ref(A, ae, W, we)
    ref128, _ = ogemm.gemm_a8w8_blockscale(A, mx.e8m0_decode(ae128).astype(np.float32), W,
                                           mx.e8m0_decode(we128).astype(np.float32))
    # the same sum with the groups summed in a different order (float64 rounding only)
    np.testing.assert_allclose(ref, ref128, rtol=1e-13, atol=1e-13 * np.abs(ref).max())


def test_batched_is_per_matrix():
    b = 3
    cases = [_raw(4, 64, 96, 20 + i) for i in range(b)]
    A, ae, W, we = (np.stack([c[j] for c in cases]) for j in range(4))
    ref, out = mx.batched_gemm_a8w8_mx32(A, ae, W, we)
    for i in range(b):
        np.testing.assert_array_equal(ref[i], mx.gemm_a8w8_mx32_ref(*cases[i]))


def test_planted_mistakes_are_caught():
    M, N, K = 3, 96, 128
    A, ae, W, we = _raw(M, N, K, 31)
    ref = mx.gemm_a8w8_mx32_ref(A, ae, W, we)
    Ad, Wd = e4m3.decode(A), e4m3.decode(W)
    sa, sw = mx.e8m0_decode(ae), mx.e8m0_decode(we)
    wrong_block = sum((sa[:, g][:, None] * sw[np.minimum(np.arange(N) // 128, sw.shape[0] - 1), g][None, :])
                      * (Ad[:, g * 32:(g + 1) * 32] @ Wd[:, g * 32:(g + 1) * 32].T) for g in range(K // 32))
    off_by_one_bias = ref * 2.0
    wrong_group = sum((sa[:, g][:, None] * sw[np.arange(N) // 32, (g + 1) % (K // 32)][None, :])
                      * (Ad[:, g * 32:(g + 1) * 32] @ Wd[:, g * 32:(g + 1) * 32].T) for g in range(K // 32))
    for bad in (wrong_block, off_by_one_bias, wrong_group):
        assert not np.allclose(bad, ref, rtol=1e-6)
