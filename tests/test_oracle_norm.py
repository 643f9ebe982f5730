"""Pins for the oracle's fused residual add + RMSNorm + activation quantisation (CPU only)."""

import numpy as np
import torch

from oracle import norm, quant
from fp8_block_scaled_a8w8_b200 import inputs


def _case(M, K, seed):
    x = inputs.activation_bf16(M, K, seed).float().numpy()
    r = inputs.activation_bf16(M, K, seed + 1).float().numpy()
    g = (1.0 + 0.1 * inputs.activation_bf16(1, K, seed + 2).float()).to(torch.bfloat16).float().numpy()[0]
    return x, r, g


def test_residual_add_is_one_bf16_rounding_of_the_fp32_sum():
    # against torch: bf16 + bf16 computed as float32 and cast to bf16 (round to nearest even)
    x, r, _ = _case(64, 512, 1)
    want = (torch.from_numpy(x) + torch.from_numpy(r)).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(norm.add_residual(x, r), want)


def test_rmsnorm_matches_torch_float64():
    x, r, g = _case(16, 640, 3)
    h = norm.add_residual(x, r)
    want = torch.nn.functional.rms_norm(torch.from_numpy(h), (640,), torch.from_numpy(g.astype(np.float64)),
                                        eps=1e-6).numpy()
    np.testing.assert_allclose(norm.rmsnorm(h, g, 1e-6), want, rtol=1e-13, atol=0)


def test_constant_row_closed_form():
    # h = c everywhere: mean square c^2, y = c / sqrt(c^2 + eps) * gamma
    K, c, eps = 256, 3.0, 1e-6
    x = np.full((1, K), c, dtype=np.float32)
    r = np.zeros((1, K), dtype=np.float32)
    g = np.linspace(0.5, 2.0, K)
    y = norm.rmsnorm(norm.add_residual(x, r), g, eps)
    np.testing.assert_allclose(y[0], c / np.sqrt(c * c + eps) * g, rtol=1e-15)


def test_zero_row_gives_zero_codes_and_scales():
    K = 384
    x = inputs.activation_bf16(1, K, 5).float().numpy()
    h, y, q, s = norm.add_rmsnorm_quant(x, -x, np.ones(K), 1e-6)
    assert np.all(h == 0) and np.all(y == 0)
    assert np.all(s == 0) and np.all(q == 0x00)


def test_quant_step_is_the_activation_quantiser_on_float32_y():
    x, r, g = _case(8, 1024, 7)
    h, y, q, s = norm.add_rmsnorm_quant(x, r, g, 1e-6)
    q2, s2 = quant.quant_act_per_token_group(y.astype(np.float32))
    np.testing.assert_array_equal(q, q2)
    np.testing.assert_array_equal(s, s2)
    # and every group's largest |y| encodes to +-448 (the scale definition)
    for gi in range(1024 // 128):
        blk = np.abs(y[:, gi * 128:(gi + 1) * 128].astype(np.float32))
        j = np.argmax(blk, axis=1)
        assert np.all((q[np.arange(8), gi * 128 + j] & 0x7F) == 0x7E)


def test_planted_mistakes_are_caught():
    x, r, g = _case(4, 512, 9)
    h = norm.add_residual(x, r)
    good = norm.rmsnorm(h, g, 1e-6)
    no_eps = h / np.sqrt(np.mean(h * h, axis=1, keepdims=True)) * g
    wrong_mean = h / np.sqrt(np.sum(h * h, axis=1, keepdims=True) / 511 + 1e-6) * g
    unrounded = (x.astype(np.float64) + r) / np.sqrt(np.mean((x.astype(np.float64) + r) ** 2, axis=1,
                                                             keepdims=True) + 1e-6) * g
    ref = torch.nn.functional.rms_norm(torch.from_numpy(h), (512,), torch.from_numpy(g.astype(np.float64)),
                                       eps=1e-6).numpy()
    np.testing.assert_allclose(good, ref, rtol=1e-13)
    for bad in (wrong_mean, unrounded):
        assert np.max(np.abs(bad - ref) / np.abs(ref).max()) > 1e-4
    # eps matters only at rows of tiny mean square: a row scaled by 1e-4 exposes it
    hs = h * 1e-4
    assert np.max(np.abs(norm.rmsnorm(hs, g, 1e-6) - hs / np.sqrt(np.mean(hs * hs, axis=1, keepdims=True)) * g)) > 1e-3
    del no_eps
