"""Tiled weight layout (fp8bs_tile_weight_e4m3 + FP8BS_FLAG_TILED_WEIGHTS).

The tiling is a byte permutation, checked byte for byte against its definition written out
here: tile (b, g) at (b * K/128 + g) * 16384, row r's 16-byte chunk c at chunk c ^ (r % 8),
rows past N and the padding block zero. A GEMM on the tiled copy runs the same kernel
arithmetic as on [N, K] (only the weight copy differs), so its output must equal the
standard-layout call of the same configuration bit for bit; and the oracle's within the
GEMM tolerance."""

import numpy as np
import pytest
import torch

import fp8_block_scaled_a8w8_b200 as fb
from fp8_block_scaled_a8w8_b200 import inputs
from oracle import quant as oquant
from tests.helpers import bf16_bits, check_a8w8, codes_to_device

pytestmark = pytest.mark.gpu
OP = fb.OP_A8W8_BLOCKSCALE


def _tiled_reference(W: np.ndarray) -> np.ndarray:
    N, K = W.shape
    G = K // 128
    nblk = (N + 127) // 128
    nblk += nblk % 2
    out = np.zeros(nblk * G * 16384, dtype=np.uint8)
    for b in range(nblk):
        for g in range(G):
            base = (b * G + g) * 16384
            for r in range(128):
                row = b * 128 + r
                if row >= N:
                    continue
                src = W[row, g * 128:(g + 1) * 128].reshape(8, 16)
                for c in range(8):
                    d = base + r * 128 + (c ^ (r % 8)) * 16
                    out[d:d + 16] = src[c]
    return out


@pytest.mark.parametrize("N,K", [(128, 128), (400, 1408), (130, 256), (256, 512)])
def test_tile_layout_matches_its_definition(N, K):
    W = inputs.random_e4m3_codes((N, K), seed=N + K)
    wt = fb.tile_weight(codes_to_device(W))
    torch.cuda.synchronize()
    assert wt.numel() == fb.tiled_weight_bytes(N, K)
    np.testing.assert_array_equal(wt.cpu().numpy(), _tiled_reference(W))


def _pair(M, N, K, seed, static=False):
    x = inputs.activation_bf16(M, K, seed).cuda()
    w = inputs.weight_f32(N, K, seed + 1).cuda()
    wq, ws = fb.quant_weight_block128(w)
    q, s = fb.quant_act_per_token_group(x)
    wt = fb.tile_weight(wq)
    y_std = fb.gemm_a8w8_blockscale(q, s, wq, ws, static_weights=static)
    y_til = fb.gemm_a8w8_blockscale(q, s, wt, ws, static_weights=static, tiled_weights=True, N=N)
    torch.cuda.synchronize()
    assert fb.get_device_status() == 0
    return y_std, y_til, (q, s, wq, ws)


@pytest.mark.parametrize("M", [1, 5, 16, 17, 32])
@pytest.mark.parametrize("N,K", [(5120, 6144), (400, 1408), (1040, 1152)])
def test_decode_tiled_equals_standard(M, N, K):
    _, cfg = fb.dispatch_lookup(OP, M, N, K)
    assert cfg == "a8w8_gemv_umma"
    for static in (False, True):
        y_std, y_til, _ = _pair(M, N, K, seed=M * 7 + N, static=static)
        assert np.array_equal(bf16_bits(y_std), bf16_bits(y_til))


@pytest.mark.parametrize("M,N,K", [(48, 400, 1408), (300, 640, 512), (130, 5120, 6144), (2048, 14336, 5120),
                                   (257, 1040, 1152)])
def test_prefill_tiled_equals_standard(M, N, K):
    fb.dispatch_reset_table(keep_builtin=False)  # the default (wide-epilogue) configuration on both calls
    try:
        _, cfg = fb.dispatch_lookup(OP, M, N, K)
        assert cfg.startswith("a8w8_tcw")
        y_std, y_til, _ = _pair(M, N, K, seed=M + N)
    finally:
        fb.dispatch_reset_table(keep_builtin=True)
    assert np.array_equal(bf16_bits(y_std), bf16_bits(y_til))


@pytest.mark.parametrize("cfg", ["a8w8_tcw_bn128", "a8w8_tcw_bn256", "a8w8_tcw_bn128_sk4", "a8w8_tcw_bn256_sk2"])
def test_every_wide_configuration_reads_tiles(cfg):
    M, N, K = 96, 768, 2048
    fb.dispatch_set_row(OP, M, N, K, cfg)
    try:
        y_std, y_til, _ = _pair(M, N, K, seed=3)
    finally:
        fb.dispatch_reset_table(keep_builtin=True)
    assert np.array_equal(bf16_bits(y_std), bf16_bits(y_til))


@pytest.mark.parametrize("M,forced", [(4, "a8w8_gemv_tma"), (64, "a8w8_tc_bn128"), (64, "a8w8_tc2_bn256")])
def test_rows_naming_other_kernels_run_the_default(M, forced):
    N, K = 1024, 1024
    x = inputs.activation_bf16(M, K, 9).cuda()
    wq, ws = fb.quant_weight_block128(inputs.weight_f32(N, K, 10).cuda())
    q, s = fb.quant_act_per_token_group(x)
    wt = fb.tile_weight(wq)
    fb.dispatch_reset_table(keep_builtin=False)
    y_default = fb.gemm_a8w8_blockscale(q, s, wq, ws)
    fb.dispatch_set_row(OP, M, N, K, forced)
    try:
        y_til = fb.gemm_a8w8_blockscale(q, s, wt, ws, tiled_weights=True, N=N)
        torch.cuda.synchronize()
    finally:
        fb.dispatch_reset_table(keep_builtin=True)
    assert np.array_equal(bf16_bits(y_default), bf16_bits(y_til))


def test_decode_shape_without_staged_scales_is_unsupported():
    M, N, K = 32, 256, 16384  # the scales do not fit the decode kernel's staging region
    q = codes_to_device(inputs.random_e4m3_codes((M, K), 1))
    s = torch.ones(M, K // 128, device="cuda")
    wt = torch.zeros(fb.tiled_weight_bytes(N, K), dtype=torch.uint8, device="cuda")
    ws = torch.ones((N + 127) // 128, K // 128, device="cuda")
    with pytest.raises(fb.Fp8bsError):
        fb.gemm_a8w8_blockscale(q, s, wt, ws, tiled_weights=True, N=N)


def test_tiled_against_the_oracle():
    M, N, K = 9, 5120, 6144
    x = inputs.activation_bf16(M, K, 41, outliers=True)
    w = inputs.weight_f32(N, K, 42)
    wq, ws = fb.quant_weight_block128(w.cuda())
    q, s = fb.quant_act_per_token_group(x.cuda())
    y = fb.gemm_a8w8_blockscale(q, s, fb.tile_weight(wq), ws, tiled_weights=True, N=N)
    torch.cuda.synchronize()
    # the oracle's own chain from the same float inputs
    A_q, a_s = oquant.quant_act_per_token_group(x.float().numpy())
    W_q, w_s = oquant.quant_weight_block128(w.numpy())
    check_a8w8(y, A_q, a_s, W_q, w_s)
