"""The allocation-free decode GEMM entry point (fp8bs_gemm_a8w8_blockscale_noalloc).

It exists for callers that cannot allocate device memory where they issue a GEMM (a fixed
or externally owned memory pool, or a place where an allocation would synchronise), so it
takes its scratch from an array in the library image instead of a workspace. Here it is
called through the C ABI and compared with the workspace entry point's output, within the
parity tolerance, on two calls in a row (the second reuses what the first left in the
shared array). The file sorts last so that a run stopping at the first failure has already
run every other test; it also passes on its own in a fresh process.
"""

import numpy as np
import pytest
import torch

import fp8_block_scaled_a8w8_b200 as fb
from fp8_block_scaled_a8w8_b200 import inputs
from oracle import metrics as ometrics
from tests.helpers import REL_L2_TOL, check_a8w8, codes_to_device

pytestmark = pytest.mark.gpu


def _case(M, N, K, seed):
    A_q = inputs.random_e4m3_codes((M, K), seed)
    W_q = inputs.random_e4m3_codes((N, K), seed + 1)
    a_s = inputs.random_scales((M, K // 128), seed + 2)
    w_s = inputs.random_scales(((N + 127) // 128, K // 128), seed + 3)
    dev = (codes_to_device(A_q), torch.from_numpy(a_s).cuda(), codes_to_device(W_q), torch.from_numpy(w_s).cuda())
    return (A_q, a_s, W_q, w_s), dev


def _noalloc(A, a_s, W, w_s):
    M, K = A.shape
    N = W.shape[0]
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    st = fb.lib().fp8bs_gemm_a8w8_blockscale_noalloc(A.data_ptr(), a_s.data_ptr(), W.data_ptr(), w_s.data_ptr(),
                                                     out.data_ptr(), M, N, K,
                                                     torch.cuda.current_stream().cuda_stream)
    assert st == 0, fb.status_string(st)
    return out


@pytest.mark.parametrize("calls", [[(1, 5120, 6144), (16, 34816, 5120)], [(9, 2048, 1024), (3, 272, 640)]])
def test_noalloc_matches_workspace_entry_point(calls):
    for i, (M, N, K) in enumerate(calls):  # two calls in a row sharing the library's scratch array
        host, dev = _case(M, N, K, seed=40 + 7 * i + M)
        y_ref = fb.gemm_a8w8_blockscale(*dev)
        y = _noalloc(*dev)
        torch.cuda.synchronize()
        assert fb.get_device_status() == 0
        rl = ometrics.rel_l2(y.float().cpu().numpy(), y_ref.float().cpu().numpy())
        assert rl <= REL_L2_TOL, rl
        check_a8w8(y, *host)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    _, dev = _case(40, 256, 256, seed=1)  # M above the decode limit of 32
    out = torch.empty((40, 256), dtype=torch.bfloat16, device="cuda")
    A, a_s, W, w_s = dev
    st = fb.lib().fp8bs_gemm_a8w8_blockscale_noalloc(A.data_ptr(), a_s.data_ptr(), W.data_ptr(), w_s.data_ptr(),
                                                     out.data_ptr(), 40, 256, 256,
                                                     torch.cuda.current_stream().cuda_stream)
    assert st == 2  # FP8BS_ERR_UNSUPPORTED, nothing launched
