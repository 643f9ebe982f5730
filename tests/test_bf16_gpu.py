"""bf16 small-N GEMM kernels vs the oracle."""

import numpy as np
import pytest
import torch

import fp8_block_scaled_a8w8_b200 as fb
from fp8_block_scaled_a8w8_b200 import inputs
from tests.helpers import check_bf16

pytestmark = pytest.mark.gpu
OP = fb.OP_BF16


def _run(M, N, K, out_fp32, seed, cfg=None):
    A = inputs.activation_bf16(M, K, seed)
    W = inputs.weight_bf16(N, K, seed + 1)
    if cfg:
        fb.dispatch_set_row(OP, M, N, K, cfg)
    try:
        y = fb.gemm_bf16(A.cuda(), W.cuda(), out_fp32=out_fp32)
        torch.cuda.synchronize()
        assert fb.get_device_status() == 0
    finally:
        if cfg:
            fb.dispatch_reset_table(True)
    return y, A.float().numpy(), W.float().numpy()


@pytest.mark.parametrize("M", [1, 3, 16, 17, 32, 33, 130, 576])
@pytest.mark.parametrize("N,K,out_fp32", [(256, 6144, False), (32, 6144, False), (384, 5120, False),
                                          (1024, 5120, True), (128, 512, False), (48, 192, False)])
def test_bf16_parity(M, N, K, out_fp32):
    y, A, W = _run(M, N, K, out_fp32, seed=M + N)
    check_bf16(y, A, W, out_fp32)


@pytest.mark.parametrize("cfg", ["bf16_tc_bn32", "bf16_tc_bn64", "bf16_tc_bn128", "bf16_tc_bn192", "bf16_tc_bn256",
                                 "bf16_gemv_d2", "bf16_gemv_d4", "bf16_gemv_umma"])
def test_bf16_configs(cfg):
    M = 20 if "gemv" in cfg else 200
    y, A, W = _run(M, 384, 640, False, seed=5, cfg=cfg)
    check_bf16(y, A, W, False)


@pytest.mark.parametrize("M,N,K,out_fp32", [(1, 1024, 5120, True), (9, 144, 1344, False), (32, 4096, 64, True),
                                            (5, 16, 6144, False)])
def test_bf16_weight_streaming_tcgen05(M, N, K, out_fp32):
    """The tcgen05 weight-streaming kernel: fp32 and bf16 out, N tails inside a 128-row block,
    a single 64-column chunk, and a weight small enough that few CTAs share it; two calls
    in a row give the same bits (fixed-order split-K sums)."""
    y, A, W = _run(M, N, K, out_fp32, seed=M + 3, cfg="bf16_gemv_umma")
    check_bf16(y, A, W, out_fp32)
    y2, _, _ = _run(M, N, K, out_fp32, seed=M + 3, cfg="bf16_gemv_umma")
    assert torch.equal(y.view(torch.int16) if not out_fp32 else y.view(torch.int32),
                       y2.view(torch.int16) if not out_fp32 else y2.view(torch.int32))


@pytest.mark.parametrize("M", [4096, 16384])
@pytest.mark.parametrize("N,K,out_fp32", [(256, 6144, False), (1024, 5120, True)])
def test_bf16_full_size_sampled_rows(M, N, K, out_fp32):
    y, A, W = _run(M, N, K, out_fp32, seed=9)
    rows = np.unique(np.concatenate([[0, 127, 128, M - 1], np.random.default_rng(M).choice(M, 12, replace=False)]))
    check_bf16(y, A, W, out_fp32, rows=rows)


_LM = {}


@pytest.mark.parametrize("M", inputs.LM_HEAD_MS)
def test_lm_head_full_size_sampled_rows(M):
    """The large-N bf16 lm_head (N = 32320, K = 5120: the last 256-column tile is ragged)
    at the M values the pages measure, on 48 rows: first and last rows, both sides of
    128-row tile boundaries, seeded random rows."""
    N, K = inputs.LM_HEAD_NK
    if "W" not in _LM:
        _LM["W"] = inputs.weight_bf16(N, K, 41)
        _LM["Wd"] = _LM["W"].cuda()
    A = inputs.activation_bf16(M, K, 42 + M)
    y = fb.gemm_bf16(A.cuda(), _LM["Wd"])
    torch.cuda.synchronize()
    assert fb.get_device_status() == 0
    rng = np.random.default_rng(M)
    fixed = [0, 1, M - 1] + [t for b in range(128, M, 128) for t in (b - 1, b)][:16]
    rows = np.unique(np.concatenate([fixed, rng.choice(M, min(M, 48 - len(fixed)), replace=False)]))
    check_bf16(y, A.float().numpy(), _LM["W"].float().numpy(), False, rows=rows)
