"""The failure path of the bounded device-side waits, made to run without any fault.

The testing hook fp8bs_test_set_wait_fault shortens every wait of the tensor-core a8w8
kernels (configurations a8w8_tcw_* and the CTA-pair a8w8_tc2_*) to 20 ms and has CTA 0's
producer leave one K group's stage unfilled, so the MMA issuer's wait on that stage runs
out (with CTA pairs the peer's waits then run out on their own). The kernel must give up,
drain what it issued, free its tensor memory and return; the host then reads
FP8BS_ERR_TIMEOUT from fp8bs_get_device_status, and the next call -- on a re-zeroed
workspace, with the hook cleared -- must be correct against the oracle.
"""

import time

import numpy as np
import pytest
import torch

import fp8_block_scaled_a8w8_b200 as fb
from fp8_block_scaled_a8w8_b200 import inputs
from tests.helpers import check_a8w8, codes_to_device

pytestmark = pytest.mark.gpu
OP = fb.OP_A8W8_BLOCKSCALE
TIMEOUT = 6  # FP8BS_ERR_TIMEOUT


@pytest.mark.parametrize("M,N,K,cfg,skip", [
    (1024, 2560, 1024, "a8w8_tcw_bn256", 3),   # 80 tiles, no split K
    (256, 1024, 2048, "a8w8_tcw_bn128", 1),    # 16 tiles x 8 K splits
    (1000, 2560, 1024, "a8w8_tcw_bn128", 0),   # the very first stage
    (2048, 4864, 1024, "a8w8_tc2_bn256", 3),   # CTA pairs: the leader's stage 3
    (300, 512, 512, "a8w8_tc2_bn256", 0),      # CTA pairs, a single pair tile
    (2048, 4864, 1024, "a8w8_tc2h_bn256", 5),  # CTA pairs, two MMA halves per K step
])
def test_wait_runs_out_reports_timeout_and_recovers(M, N, K, cfg, skip):
    A_q = inputs.random_e4m3_codes((M, K), 1)
    W_q = inputs.random_e4m3_codes((N, K), 2)
    a_s = inputs.random_scales((M, K // 128), 3)
    w_s = inputs.random_scales(((N + 127) // 128, K // 128), 4)
    A, W = codes_to_device(A_q), codes_to_device(W_q)
    sa, sw = torch.from_numpy(a_s).cuda(), torch.from_numpy(w_s).cuda()
    fb.dispatch_set_row(OP, M, N, K, cfg)
    ws = torch.zeros(max(256, fb.workspace_bytes(OP, M, N, K)), dtype=torch.uint8, device="cuda")
    out = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
    try:
        assert fb.get_device_status() == 0
        fb.test_set_wait_fault(20_000_000, skip)
        t0 = time.time()
        fb.gemm_a8w8_blockscale(A, sa, W, sw, out=out, workspace=ws)
        st = fb.get_device_status()  # synchronises
        elapsed = time.time() - t0
        fb.test_set_wait_fault(0, -1)
        assert st == TIMEOUT, st
        assert elapsed < 5.0, elapsed
        assert fb.get_device_status() == 0  # the status word was cleared by the read
        # the context is still usable: re-zero the workspace and run again, hook cleared
        ws.zero_()
        y = fb.gemm_a8w8_blockscale(A, sa, W, sw, out=out, workspace=ws)
        assert fb.get_device_status() == 0
        check_a8w8(y, A_q, a_s, W_q, w_s)
    finally:
        fb.test_set_wait_fault(0, -1)
        fb.dispatch_reset_table(True)


def test_hook_rejects_bad_iteration():
    with pytest.raises(fb.Fp8bsError):
        fb.test_set_wait_fault(0, -2)
    fb.test_set_wait_fault(0, -1)
