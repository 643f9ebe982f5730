"""Pins for the oracle's GEMMs and metrics (CPU only).

Each pin checks the oracle against something other than itself: exact
rational arithmetic, integer arithmetic, algebraic invariants, a plain matmul
in another library, and the accuracy floor the pages print. The last test
plants plausible mistakes in copies of the oracle and checks that the pins
catch each one.
"""

from fractions import Fraction
import os

import numpy as np
import pytest
import torch

from oracle import bf16, e4m3, gemm, metrics, quant
from fp8_block_scaled_a8w8_b200 import inputs


def _exact_a8w8(A_q, a_s, W_q, w_s):
    """Brute force with exact rationals, straight from the definition."""
    M, K = A_q.shape
    N = W_q.shape[0]
    dec = [Fraction(float(e4m3.decode_code(c))) if c not in (0x7F, 0xFF) else None for c in range(256)]
    out = [[Fraction(0)] * N for _ in range(M)]
    for m in range(M):
        for n in range(N):
            tot = Fraction(0)
            for g in range(K // 128):
                part = Fraction(0)
                for k in range(g * 128, (g + 1) * 128):
                    part += dec[int(A_q[m, k])] * dec[int(W_q[n, k])]
                tot += Fraction(float(a_s[m, g])) * Fraction(float(w_s[n // 128, g])) * part
            out[m][n] = tot
    return out


def _tiny_case(seed, M=2, N=136, K=256):
    A_q = inputs.random_e4m3_codes((M, K), seed)
    W_q = inputs.random_e4m3_codes((N, K), seed + 1)
    a_s = inputs.random_scales((M, K // 128), seed + 2)
    w_s = inputs.random_scales(((N + 127) // 128, K // 128), seed + 3)
    return A_q, a_s, W_q, w_s


def _check_against_exact(fn, case):
    A_q, a_s, W_q, w_s = case
    ref = fn(A_q, a_s, W_q, w_s)
    exact = _exact_a8w8(A_q, a_s, W_q, w_s)
    ex = np.array([[float(v) for v in row] for row in exact])
    ok_ref = np.allclose(ref, ex, rtol=1e-13, atol=1e-300)
    # rounding the exact rational to bf16 must agree with the oracle's bf16 output
    out_bf16 = bf16.round_to_bf16(ref)
    ok_bf16 = np.array_equal(out_bf16, bf16.round_to_bf16(ex))
    return ok_ref and ok_bf16


@pytest.mark.parametrize("seed", [1, 2])
def test_exact_rational_brute_force(seed):
    assert _check_against_exact(gemm.gemm_a8w8_blockscale_ref, _tiny_case(seed))


def test_integer_valued_exact():
    """Integer-valued e4m3 codes (|v| <= 4) and power-of-two scales: the result is an
    exact dyadic rational that int64 arithmetic reproduces."""
    rng = np.random.default_rng(21)
    M, N, K = 5, 260, 512
    int_codes = {0: 0x00, 1: 0x38, 2: 0x40, 3: 0x44, 4: 0x48}
    Ai = rng.integers(-4, 5, size=(M, K))
    Wi = rng.integers(-4, 5, size=(N, K))
    enc = lambda v: np.vectorize(lambda x: int_codes[abs(x)] | (0x80 if x < 0 else 0))(v).astype(np.uint8)
    A_q, W_q = enc(Ai), enc(Wi)
    G = K // 128
    ae = rng.integers(-6, 3, size=(M, G))
    we = rng.integers(-6, 3, size=((N + 127) // 128, G))
    a_s = np.ldexp(1.0, ae).astype(np.float32)
    w_s = np.ldexp(1.0, we).astype(np.float32)
    ref = gemm.gemm_a8w8_blockscale_ref(A_q, a_s, W_q, w_s)
    # integer arithmetic with a common power-of-two denominator 2^12
    want = np.zeros((M, N), dtype=np.int64)
    for g in range(G):
        ks = slice(g * 128, (g + 1) * 128)
        P = Ai[:, ks].astype(np.int64) @ Wi[:, ks].T.astype(np.int64)
        sh = ae[:, g][:, None] + we[np.arange(N) // 128, g][None, :] + 12
        want += P << sh
    assert np.array_equal(ref, np.ldexp(want.astype(np.float64), -12))


def test_scale_linearity():
    A_q, a_s, W_q, w_s = _tiny_case(5, M=4, N=300, K=512)
    base = gemm.gemm_a8w8_blockscale_ref(A_q, a_s, W_q, w_s)
    a2 = a_s.copy(); a2[2, :] *= 2
    r = gemm.gemm_a8w8_blockscale_ref(A_q, a2, W_q, w_s)
    assert np.array_equal(r[2], 2 * base[2]) and np.array_equal(np.delete(r, 2, 0), np.delete(base, 2, 0))
    w2 = w_s.copy(); w2[1, :] *= 2
    r = gemm.gemm_a8w8_blockscale_ref(A_q, a_s, W_q, w2)
    assert np.array_equal(r[:, 128:256], 2 * base[:, 128:256])
    assert np.array_equal(r[:, :128], base[:, :128]) and np.array_equal(r[:, 256:], base[:, 256:])
    # changing one group's scale moves row m by (new - old) scale times that group's partial
    c = np.float32(3.0)
    a3 = a_s.copy(); a3[1, 2] *= c
    r = gemm.gemm_a8w8_blockscale_ref(A_q, a3, W_q, w_s)
    ks = slice(256, 384)
    Pg = e4m3.decode(A_q[1, ks]) @ e4m3.decode(W_q[:, ks]).T
    delta = (float(a3[1, 2]) - float(a_s[1, 2])) * w_s[np.arange(300) // 128, 2].astype(np.float64) * Pg
    np.testing.assert_allclose(r[1] - base[1], delta, rtol=1e-9, atol=1e-12 * np.abs(base[1]).max())


def test_permutation_within_group_invariant():
    A_q, a_s, W_q, w_s = _tiny_case(6, M=3, N=128, K=384)
    perm = np.concatenate([g * 128 + np.random.default_rng(g).permutation(128) for g in range(3)])
    r1 = gemm.gemm_a8w8_blockscale_ref(A_q, a_s, W_q, w_s)
    r2 = gemm.gemm_a8w8_blockscale_ref(A_q[:, perm], a_s, W_q[:, perm], w_s)
    np.testing.assert_allclose(r1, r2, rtol=1e-14, atol=0)


def test_unit_scales_reduce_to_plain_matmul():
    A_q, _, W_q, _ = _tiny_case(9, M=7, N=256, K=640)
    ones_a = np.ones((7, 5), np.float32)
    ones_w = np.ones((2, 5), np.float32)
    r = gemm.gemm_a8w8_blockscale_ref(A_q, ones_a, W_q, ones_w)
    A = torch.from_numpy(A_q.copy()).view(torch.float8_e4m3fn).to(torch.float64)
    W = torch.from_numpy(W_q.copy()).view(torch.float8_e4m3fn).to(torch.float64)
    np.testing.assert_array_equal(r, (A @ W.T).numpy())  # both exact in float64


def test_bf16_rounding_floor_matches_pages(golden_dir):
    """relL2(bf16(ref), ref) on the decode distributions reproduces the page's floor."""
    floor = dict(l.split() for l in open(os.path.join(golden_dir, "accuracy_floor.txt"))
                 if l.strip() and not l.startswith("#"))
    page = float(floor["bf16_output_rounding_floor"])
    x, w = inputs.m1_n5120_k6144(0)
    A_q, a_s = quant.quant_act_per_token_group(x.float().numpy())
    W_q, w_s = quant.quant_weight_block128(w.numpy())
    ref, out = gemm.gemm_a8w8_blockscale(A_q, a_s, W_q, w_s)
    rl = metrics.rel_l2(out, ref)
    assert abs(rl - page) / page < 0.15, rl


def test_bf16_gemm_exact_and_matmul():
    rng = np.random.default_rng(4)
    A = rng.integers(-8, 9, size=(6, 512)).astype(np.float64)
    W = rng.integers(-8, 9, size=(40, 512)).astype(np.float64)
    ref, out = gemm.gemm_bf16(A, W)
    assert np.array_equal(ref, (A.astype(np.int64) @ W.T.astype(np.int64)).astype(np.float64))
    Ab = inputs.activation_bf16(5, 512, 1)
    Wb = inputs.weight_bf16(33, 512, 2)
    ref, out32 = gemm.gemm_bf16(Ab.float().numpy(), Wb.float().numpy(), out_fp32=True)
    th = (Ab.double() @ Wb.double().T).numpy()
    np.testing.assert_allclose(ref, th, rtol=1e-12, atol=1e-15)
    assert np.array_equal(out32, th.astype(np.float32).astype(np.float64))
    # exact rational brute force on a tiny case
    a = Ab.float().numpy()[:2, :128]
    b = Wb.float().numpy()[:3, :128]
    r, _ = gemm.gemm_bf16(a, b)
    for i in range(2):
        for j in range(3):
            ex = sum(Fraction(float(a[i, k])) * Fraction(float(b[j, k])) for k in range(128))
            assert abs(r[i, j] - float(ex)) <= 1e-15 * max(1.0, abs(float(ex)))


# ---- plant-a-mistake: each mutated oracle must fail at least one pin ----------------

def _mut_wscale_modulo(A_q, a_s, W_q, w_s):
    A, W = e4m3.decode(A_q), e4m3.decode(W_q)
    out = np.zeros((A.shape[0], W.shape[0]))
    nb = np.arange(W.shape[0]) % w_s.shape[0]  # wrong: n % NB instead of n // 128
    for g in range(A.shape[1] // 128):
        ks = slice(g * 128, (g + 1) * 128)
        out += a_s[:, g][:, None].astype(np.float64) * w_s[nb, g][None, :] * (A[:, ks] @ W[:, ks].T)
    return out


def _mut_drop_last_group(A_q, a_s, W_q, w_s):
    return gemm.gemm_a8w8_blockscale_ref(A_q[:, :-128], a_s[:, :-1], W_q[:, :-128], w_s[:, :-1])


def _mut_swapped_group_scales(A_q, a_s, W_q, w_s):
    return gemm.gemm_a8w8_blockscale_ref(A_q, a_s[:, ::-1].copy(), W_q, w_s)


def _mut_sign_dropped(A_q, a_s, W_q, w_s):
    return gemm.gemm_a8w8_blockscale_ref(A_q & 0x7F, a_s, W_q, w_s)


def _mut_transposed_w_rows(A_q, a_s, W_q, w_s):
    r = gemm.gemm_a8w8_blockscale_ref(A_q, a_s, W_q, w_s)
    return r[:, ::-1]


@pytest.mark.parametrize("mut", [_mut_wscale_modulo, _mut_drop_last_group, _mut_swapped_group_scales,
                                 _mut_sign_dropped, _mut_transposed_w_rows])
def test_planted_mistakes_are_caught(mut):
    assert not _check_against_exact(mut, _tiny_case(1))
