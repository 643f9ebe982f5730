"""Fused residual add + RMSNorm + activation quantisation on the GPU vs the oracle.

residual_out must equal the oracle's h bit for bit. The quantiser works on y, which the
kernel computes with a float32 mean square and the oracle in float64, so a scale may
differ in its last bits and a code may sit one step away where the oracle's y / scale is
within float32 error of a rounding midpoint; those codes are checked to be the
neighbouring one at such a midpoint, every other code must be equal.
"""

import numpy as np
import pytest
import torch

import fp8_block_scaled_a8w8_b200 as fb
from fp8_block_scaled_a8w8_b200 import inputs
from oracle import e4m3 as oe4m3
from oracle import norm as onorm
from tests.helpers import codes_from_device

pytestmark = pytest.mark.gpu
EPS = 1e-6


def _inputs(M, K, seed):
    x = inputs.activation_bf16(M, K, seed)
    r = inputs.activation_bf16(M, K, seed + 1)
    g = (1.0 + 0.1 * inputs.activation_bf16(1, K, seed + 2).float()).to(torch.bfloat16)[0]
    return x, r, g


def _check(x, r, g, res_out, q, s):
    h, y, Aq, As = onorm.add_rmsnorm_quant(x.float().numpy(), r.float().numpy(), g.float().numpy(), EPS)
    # the residual stream: exact
    assert np.array_equal(res_out.float().cpu().numpy().astype(np.float64), h)
    sg = s.cpu().numpy()
    assert np.all(np.abs(sg - As) <= 2.0 ** -18 * As), "scales"
    qg = codes_from_device(q)
    bad = qg != Aq
    if bad.any():
        assert bad.mean() < 1e-3, bad.mean()
        M, K = qg.shape
        idx = np.argwhere(bad)
        for m, k in idx:
            t = np.float32(y[m, k]) / As[m, k // 128]   # the oracle's quantiser input
            a, b = oe4m3.decode(np.array([Aq[m, k], qg[m, k]], dtype=np.uint8))
            mid = (a + b) / 2.0
            assert abs(int(Aq[m, k] & 0x7F) - int(qg[m, k] & 0x7F)) == 1, (m, k)
            assert abs(t - mid) <= 1e-5 * abs(t) + 1e-30, (m, k, t, a, b)


@pytest.mark.parametrize("M,K", [(1, 128), (3, 384), (16, 5120), (130, 6144), (1000, 1024), (8, 8192), (300, 6144),
                                 (257, 8192)])
def test_add_rmsnorm_quant_parity(M, K):
    x, r, g = _inputs(M, K, M + K)
    res_out, q, s = fb.add_rmsnorm_quant(x.cuda(), r.cuda(), g.cuda(), EPS)
    torch.cuda.synchronize()
    _check(x, r, g, res_out, q, s)


def test_in_place_residual_and_zero_rows():
    M, K = 64, 640
    x, r, g = _inputs(M, K, 7)
    x[5] = -r[5]  # h = 0: scale 0, codes 0
    x[40] = -r[40]
    rd = r.cuda()
    res_out, q, s = fb.add_rmsnorm_quant(x.cuda(), rd, g.cuda(), EPS, residual_out=rd)
    torch.cuda.synchronize()
    assert res_out.data_ptr() == rd.data_ptr()
    _check(x, r, g, res_out, q, s)
    assert float(s[5].abs().max()) == 0.0 and int(codes_from_device(q)[40].max()) == 0


def test_outlier_rows_large_values():
    M, K = 32, 5120
    x = inputs.activation_bf16(M, K, 11, outliers=True)
    r = inputs.activation_bf16(M, K, 12, outliers=True)
    g = (1.0 + 0.1 * inputs.activation_bf16(1, K, 13).float()).to(torch.bfloat16)[0]
    res_out, q, s = fb.add_rmsnorm_quant(x.cuda(), r.cuda(), g.cuda(), EPS)
    torch.cuda.synchronize()
    _check(x, r, g, res_out, q, s)


def test_chain_into_the_gemm():
    """Fused step then GEMM on the GPU against the oracle's own chain (its own codes and
    scales), within the GEMM tolerance."""
    from oracle import quant as oquant
    from tests.helpers import check_a8w8
    M, K, N = 9, 5120, 1024
    x, r, g = _inputs(M, K, 21)
    w = inputs.weight_f32(N, K, 22)
    res_out, q, s = fb.add_rmsnorm_quant(x.cuda(), r.cuda(), g.cuda(), EPS)
    wq, ws = fb.quant_weight_block128(w.cuda())
    y = fb.gemm_a8w8_blockscale(q, s, wq, ws)
    torch.cuda.synchronize()
    _, _, Aq, As = onorm.add_rmsnorm_quant(x.float().numpy(), r.float().numpy(), g.float().numpy(), EPS)
    W_q, w_s = oquant.quant_weight_block128(w.numpy())
    check_a8w8(y, Aq, As, W_q, w_s)
