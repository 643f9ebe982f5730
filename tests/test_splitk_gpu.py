"""Split-K finish of the tensor-core kernels (a8w8 wide-epilogue, a8w8/bf16 two-buffer and
MX32 kernels).

A split-K launch stores one float32 partial tile per (tile, K split) and then sums every
output element's partials in split order. With one item per CTA the splits of a tile wait
for each other and each sums its own share of the tile (distributed); a persistent launch
with more items than CTAs lets the last split to arrive sum the whole tile. Both ways are
checked against the oracle, for bit-identical repeats on a reused workspace, and for the
per-tile counters (the first 256 KiB of the workspace) being back at zero after the call,
which the next call on the same workspace relies on.
"""

import re

import numpy as np
import pytest
import torch

import fp8_block_scaled_a8w8_b200 as fb
from fp8_block_scaled_a8w8_b200 import inputs
from tests.helpers import bf16_bits, check_a8w8, check_bf16, check_mx32, codes_to_device

pytestmark = pytest.mark.gpu
COUNTER_BYTES = 65536 * 4
SMS = None


def _sms():
    global SMS
    if SMS is None:
        SMS = torch.cuda.get_device_properties(0).multi_processor_count
    return SMS


def _counters_zero(ws):
    torch.cuda.synchronize()
    return int(torch.count_nonzero(ws[:COUNTER_BYTES])) == 0


def _a8w8(M, N, K, seed):
    A_q = inputs.random_e4m3_codes((M, K), seed)
    W_q = inputs.random_e4m3_codes((N, K), seed + 1)
    a_s = inputs.random_scales((M, K // 128), seed + 2)
    w_s = inputs.random_scales(((N + 127) // 128, K // 128), seed + 3)
    return A_q, a_s, W_q, w_s


@pytest.mark.parametrize("M,N,K,cfg,splits", [
    (48, 2048, 4096, "a8w8_tcw_bn256", 8),      # 8 tiles x 8 splits: distributed
    (100, 400, 1024, "a8w8_tcw_bn256", 4),      # ragged M and N tails, 2 tiles x 4 splits
    (40, 256, 6144, "a8w8_tcw_bn256", 8),       # one tile, 8 splits
    (48, 5120, 6144, "a8w8_tc_bn128", 3),       # two-buffer kernel, 40 tiles x 3 splits
    (256, 2560, 2048, "a8w8_tcw_bn128_sk8", 8),  # 40 tiles x 8 = 320 items: last arrival
    (256, 1024, 2048, "a8w8_tcw_bn128_sk8", 8),  # 16 tiles x 8 = 128 items: distributed
    (130, 1040, 1152, "a8w8_tcw_bn256_sk2", 2),  # 10 tiles x 2 splits, ragged tails
])
def test_a8w8_split_finish(M, N, K, cfg, splits):
    OP = fb.OP_A8W8_BLOCKSCALE
    A_q, a_s, W_q, w_s = _a8w8(M, N, K, seed=M + N)
    A, W = codes_to_device(A_q), codes_to_device(W_q)
    sa, sw = torch.from_numpy(a_s).cuda(), torch.from_numpy(w_s).cuda()
    fb.dispatch_set_row(OP, M, N, K, cfg)
    try:
        need = fb.workspace_bytes(OP, M, N, K)
        bn = int(re.search(r"bn(\d+)", cfg).group(1))
        tiles = ((M + 127) // 128) * ((N + bn - 1) // bn)
        assert need >= COUNTER_BYTES + tiles * splits * 128 * bn * 4  # room for this split count
        ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
        y1 = fb.gemm_a8w8_blockscale(A, sa, W, sw, workspace=ws)
        assert fb.get_device_status() == 0
        assert _counters_zero(ws)
        y2 = fb.gemm_a8w8_blockscale(A, sa, W, sw, workspace=ws)
        assert fb.get_device_status() == 0
        assert _counters_zero(ws)
    finally:
        fb.dispatch_reset_table(True)
    assert np.array_equal(bf16_bits(y1), bf16_bits(y2))
    check_a8w8(y1, A_q, a_s, W_q, w_s)


@pytest.mark.parametrize("M,N,K,out_fp32", [(576, 256, 6144, False), (130, 384, 5120, True), (48, 1024, 5120, False)])
def test_bf16_split_finish(M, N, K, out_fp32):
    OP = fb.OP_BF16
    A = inputs.activation_bf16(M, K, M)
    W = inputs.weight_bf16(N, K, N)
    need = fb.workspace_bytes(OP, M, N, K)
    assert need > 0  # these shapes split K
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    y1 = fb.gemm_bf16(A.cuda(), W.cuda(), out_fp32=out_fp32, workspace=ws)
    assert fb.get_device_status() == 0
    assert _counters_zero(ws)
    y2 = fb.gemm_bf16(A.cuda(), W.cuda(), out_fp32=out_fp32, workspace=ws)
    assert fb.get_device_status() == 0
    assert _counters_zero(ws)
    assert torch.equal(y1.view(torch.int32 if out_fp32 else torch.int16), y2.view(torch.int32 if out_fp32 else torch.int16))
    check_bf16(y1, A.float().numpy(), W.float().numpy(), out_fp32)


def _mx_raw(batch, M, N, K, seed):
    rng = np.random.default_rng(seed)
    shp = (batch,) if batch > 1 else ()
    A = inputs.random_e4m3_codes(shp + (M, K), seed)
    W = inputs.random_e4m3_codes(shp + (N, K), seed + 1)
    ae = rng.integers(112, 142, shp + (M, K // 32)).astype(np.uint8)
    we = rng.integers(112, 142, shp + ((N + 31) // 32, K // 32)).astype(np.uint8)
    return A, ae, W, we


@pytest.mark.parametrize("batch,M,N,K", [(1, 48, 1792, 5120), (1, 200, 960, 2048), (8, 16, 1024, 4096)])
def test_mx32_split_finish(batch, M, N, K):
    A, ae, W, we = _mx_raw(batch, M, N, K, seed=M + N)
    dev = (codes_to_device(A), torch.from_numpy(ae).cuda(), codes_to_device(W), torch.from_numpy(we).cuda())
    need = fb.mx32_workspace_bytes(batch, M, N, K)
    tiles = batch * ((M + 127) // 128) * ((N + 191) // 192)
    assert need > 0 and 2 * tiles < _sms()
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    y1 = fb.gemm_a8w8_mx32(*dev, workspace=ws)
    assert fb.get_device_status() == 0
    assert _counters_zero(ws)
    y2 = fb.gemm_a8w8_mx32(*dev, workspace=ws)
    assert fb.get_device_status() == 0
    assert _counters_zero(ws)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    if batch == 1:
        check_mx32(y1, A, ae, W, we)
    else:
        for b in range(batch):
            check_mx32(y1[b], A[b], ae[b], W[b], we[b])
