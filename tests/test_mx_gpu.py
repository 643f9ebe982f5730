"""MX32 variant on the GPU (E8M0 scales, 1x32 activation groups, 32x32 weight blocks,
hardware block-scaled MMAs) vs the oracle: quantisers bit for bit, the GEMM element by
element, dense and batched, at the shapes [aiter#7247] lists and at ragged ones."""

import numpy as np
import pytest
import torch

import fp8_block_scaled_a8w8_b200 as fb
from fp8_block_scaled_a8w8_b200 import inputs
from oracle import mx as omx
from tests.helpers import check_mx32, codes_from_device, codes_to_device

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,K,outliers", [(1, 32, False), (7, 96, False), (64, 5120, True), (1000, 1280, False)])
def test_quant_act_mx32_bit_exact(M, K, outliers):
    x = inputs.activation_bf16(M, K, M + K, outliers=outliers)
    x[0, :32] = 0.0                   # an all-zero group: code 0, codes +0
    if M > 1:
        x[1, 32:64] = 1e-37           # a group whose ratio amax / 448 is float32-subnormal
    q, e = fb.quant_act_mx32(x.cuda())
    torch.cuda.synchronize()
    Aq, Ae = omx.quant_act_mx32(x.float().numpy())
    np.testing.assert_array_equal(codes_from_device(q), Aq)
    np.testing.assert_array_equal(e.cpu().numpy(), Ae)


def test_quant_act_mx32_strided_rows():
    x = inputs.activation_bf16(9, 512, 3)
    q, e = fb.quant_act_mx32(x.cuda()[:, :256])  # row stride 512, K = 256
    Aq, Ae = omx.quant_act_mx32(x.float().numpy()[:, :256])
    np.testing.assert_array_equal(codes_from_device(q), Aq)
    np.testing.assert_array_equal(e.cpu().numpy(), Ae)


@pytest.mark.parametrize("N,K", [(32, 32), (70, 96), (1792, 5120)])
def test_quant_weight_mx32_bit_exact(N, K):
    w = inputs.weight_f32(N, K, N + K)
    q, e = fb.quant_weight_mx32(w.cuda())
    torch.cuda.synchronize()
    Wq, We = omx.quant_weight_mx32(w.numpy())
    np.testing.assert_array_equal(codes_from_device(q), Wq)
    np.testing.assert_array_equal(e.cpu().numpy(), We)


def _raw(M, N, K, seed, batch=None):
    rng = np.random.default_rng(seed)
    shp = (batch,) if batch else ()
    A = inputs.random_e4m3_codes(shp + (M, K), seed)
    W = inputs.random_e4m3_codes(shp + (N, K), seed + 1)
    ae = rng.integers(112, 142, shp + (M, K // 32)).astype(np.uint8)
    we = rng.integers(112, 142, shp + ((N + 31) // 32, K // 32)).astype(np.uint8)
    return A, ae, W, we


def _run(A, ae, W, we, ws=None):
    y = fb.gemm_a8w8_mx32(codes_to_device(A), torch.from_numpy(ae).cuda(), codes_to_device(W),
                          torch.from_numpy(we).cuda(), workspace=ws)
    torch.cuda.synchronize()
    assert fb.get_device_status() == 0
    return y


@pytest.mark.parametrize("M,N,K", [(1, 192, 128), (16, 256, 512), (48, 1792, 5120), (130, 2320, 384),
                                   (300, 4608, 512), (257, 1024, 1280), (600, 5120, 640),
                                   # 256-wide tiles (192-wide ones would need a partial second wave)
                                   (768, 5120, 512), (800, 4800, 384),
                                   # 256-wide tiles with K split three ways (192-wide: two ways)
                                   (768, 1792, 2048)])
def test_gemm_mx32_parity(M, N, K):
    case = _raw(M, N, K, M + N + K)
    check_mx32(_run(*case), *case)


def test_gemm_mx32_integer_valued_bit_exact():
    """Integer codes |v| <= 4 with scales 2^-3..2^3: every partial sum is exact, so the bf16
    output equals bf16(exact) bit for bit."""
    M, N, K = 200, 400, 1024
    rng = np.random.default_rng(5)
    codes = np.array([0x00, 0x38, 0x40, 0x44, 0x48], dtype=np.uint8)
    A = codes[rng.integers(0, 5, (M, K))] | (rng.integers(0, 2, (M, K)) << 7).astype(np.uint8)
    W = codes[rng.integers(0, 5, (N, K))] | (rng.integers(0, 2, (N, K)) << 7).astype(np.uint8)
    ae = rng.integers(124, 131, (M, K // 32)).astype(np.uint8)
    we = rng.integers(124, 131, ((N + 31) // 32, K // 32)).astype(np.uint8)
    y = _run(A, ae, W, we)
    _, want = omx.gemm_a8w8_mx32(A, ae, W, we)
    assert np.array_equal(y.float().cpu().numpy().astype(np.float64), want)


@pytest.mark.parametrize("M,N,K", [(768, 5120, 8192), (768, 32768, 1280), (768, 4608, 5120), (48, 5120, 2304)])
def test_gemm_mx32_pages_shapes_sampled_rows(M, N, K):
    """The dense MX32 shapes of [aiter#7247] at full size, from bf16 activations and float32
    weights quantised on the GPU (oracle quantises on its own), checked on 40 rows."""
    x = inputs.activation_bf16(M, K, 60 + M)
    w = inputs.weight_f32(N, K, 61 + N)
    q, e = fb.quant_act_mx32(x.cuda())
    wq, we = fb.quant_weight_mx32(w.cuda())
    y = fb.gemm_a8w8_mx32(q, e, wq, we)
    torch.cuda.synchronize()
    assert fb.get_device_status() == 0
    rng = np.random.default_rng(M + N)
    rows = np.unique(np.concatenate([[0, 127, 128, M - 1], rng.choice(M, min(M, 36), replace=False)]))
    rows = rows[rows < M]
    Aq, Ae = omx.quant_act_mx32(x.float().numpy()[rows])
    Wq, We = omx.quant_weight_mx32(w.numpy())
    check_mx32(y.cpu()[torch.from_numpy(rows)], Aq, Ae, Wq, We)


def test_batched_gemm_mx32_b8_full():
    """The batched MX32 GEMM of [aiter#7247] (b = 8, N = 1024, K = 4096) at M = 16, every
    output of every batch against the oracle."""
    b, M, N, K = 8, 16, 1024, 4096
    A, ae, W, we = _raw(M, N, K, 77, batch=b)
    y = _run(A, ae, W, we)
    assert y.shape == (b, M, N)
    for i in range(b):
        check_mx32(y[i], A[i], ae[i], W[i], we[i])


def test_gemm_mx32_deterministic_and_workspace_reuse():
    ws = torch.zeros(max(256, fb.mx32_workspace_bytes(8, 16, 1024, 4096), fb.mx32_workspace_bytes(1, 48, 1792, 5120)),
                     dtype=torch.uint8, device="cuda")
    c1 = _raw(48, 1792, 5120, 3)
    c2 = _raw(16, 1024, 4096, 4, batch=8)
    y1 = _run(*c1, ws=ws)
    y2 = _run(*c2, ws=ws)
    y1b = _run(*c1, ws=ws)
    assert torch.equal(y1.view(torch.int16), y1b.view(torch.int16))
    check_mx32(y1, *c1)
    for i in range(8):
        check_mx32(y2[i], c2[0][i], c2[1][i], c2[2][i], c2[3][i])
