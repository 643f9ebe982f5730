"""a8w8 block-scale GEMM kernels vs the oracle (both kernel paths, tails, exact cases,
determinism, graph replay, full-size configurations on sampled rows)."""

import numpy as np
import pytest
import torch

import fp8_block_scaled_a8w8_b200 as fb
from fp8_block_scaled_a8w8_b200 import inputs
from oracle import gemm as ogemm
from oracle import quant as oquant
from tests.helpers import bf16_bits, check_a8w8, codes_from_device, codes_to_device

pytestmark = pytest.mark.gpu
OP = fb.OP_A8W8_BLOCKSCALE


def _raw_case(M, N, K, seed):
    A_q = inputs.random_e4m3_codes((M, K), seed)
    W_q = inputs.random_e4m3_codes((N, K), seed + 1)
    a_s = inputs.random_scales((M, K // 128), seed + 2)
    w_s = inputs.random_scales(((N + 127) // 128, K // 128), seed + 3)
    return A_q, a_s, W_q, w_s


def _run(A_q, a_s, W_q, w_s, cfg=None):
    M, K = A_q.shape
    N = W_q.shape[0]
    if cfg is not None:
        fb.dispatch_set_row(OP, M, N, K, cfg)
    try:
        y = fb.gemm_a8w8_blockscale(codes_to_device(A_q), torch.from_numpy(a_s).cuda(), codes_to_device(W_q),
                                    torch.from_numpy(w_s).cuda())
        torch.cuda.synchronize()
        assert fb.get_device_status() == 0
    finally:
        if cfg is not None:
            fb.dispatch_reset_table(True)
    return y


GEMV_SHAPES = [(16, 128), (128, 256), (272, 640), (1040, 1152)]


@pytest.mark.parametrize("M", [1, 2, 3, 5, 8, 9, 13, 16, 17, 24, 31, 32])
@pytest.mark.parametrize("N,K", GEMV_SHAPES)
def test_gemv_path_parity(M, N, K):
    case = _raw_case(M, N, K, seed=M * 1000 + N + K)
    _, cfg = fb.dispatch_lookup(OP, M, N, K)
    assert cfg.startswith("a8w8_gemv")
    check_a8w8(_run(*case), *case)


@pytest.mark.parametrize("cfg", ["a8w8_gemv_d2", "a8w8_gemv_d3", "a8w8_gemv_d4", "a8w8_gemv_tma", "a8w8_gemv_umma"])
@pytest.mark.parametrize("M", [1, 7, 16, 25])
def test_gemv_depths(cfg, M):
    case = _raw_case(M, 400, 1408, seed=M + 77)
    check_a8w8(_run(*case, cfg=cfg), *case)


@pytest.mark.parametrize("cfg", ["a8w8_gemv_d4", "a8w8_gemv_tma", "a8w8_gemv_umma"])
@pytest.mark.parametrize("M,N,K", [(1, 16, 128), (5, 144, 128), (32, 34816, 5120), (12, 5120, 6144), (2, 130 * 16, 3968)])
def test_gemv_kernels_shapes(cfg, M, N, K):
    case = _raw_case(M, N, K, seed=M + N + K)
    check_a8w8(_run(*case, cfg=cfg), *case)


# The weight-streaming kernels stage each CTA's scales in a 24 KiB shared-memory region;
# K this large (a_scale of the token slots x K / 128 groups no longer fits) takes the
# mma.sync kernel's per-unit global-load variant (the tcgen05 kernel hands such shapes
# to it).
@pytest.mark.parametrize("cfg", ["a8w8_gemv_tma", "a8w8_gemv_umma"])
@pytest.mark.parametrize("M,N,K", [(1, 32, 98432), (8, 16, 98432), (32, 48, 24704), (17, 16, 32896)])
def test_gemv_scales_not_staged(cfg, M, N, K):
    case = _raw_case(M, N, K, seed=M + N + K + 5)
    check_a8w8(_run(*case, cfg=cfg), *case)


TC_SHAPES = [(256, 512), (384, 1024), (1280, 768)]


@pytest.mark.parametrize("M", [33, 100, 128, 129, 255, 300])
@pytest.mark.parametrize("N,K", TC_SHAPES)
def test_tc_path_parity(M, N, K):
    case = _raw_case(M, N, K, seed=M * 31 + N + K)
    _, cfg = fb.dispatch_lookup(OP, M, N, K)
    assert cfg.startswith("a8w8_tc")
    check_a8w8(_run(*case), *case)


@pytest.mark.parametrize("cfg", ["a8w8_tc_bn128", "a8w8_tc_bn256", "a8w8_tcw_bn128", "a8w8_tcw_bn256",
                                 "a8w8_tc2_bn256", "a8w8_tc2h_bn256"])
@pytest.mark.parametrize("M,N,K", [(1, 256, 128), (40, 512, 2048), (300, 1536, 640), (2, 272, 256),
                                   (1000, 2560, 1024), (777, 4112, 768)])
def test_tc_configs_any_m(cfg, M, N, K):
    """The tensor-core kernel on any M, including tiny M and N tails (a row can name it)."""
    case = _raw_case(M, N, K, seed=M + N + K)
    check_a8w8(_run(*case, cfg=cfg), *case)


@pytest.mark.parametrize("M,N,K,cfg", [(3, 272, 512, None), (16, 1024, 1024, None), (200, 512, 1024, None),
                                       (130, 384, 512, "a8w8_tc_bn128"), (64, 512, 384, "a8w8_tc_bn256"),
                                       (130, 384, 512, "a8w8_tcw_bn128"), (64, 512, 384, "a8w8_tcw_bn256"),
                                       (1100, 2816, 1024, "a8w8_tcw_bn256"), (300, 272, 512, "a8w8_tc2_bn256"),
                                       (2100, 4864, 1024, "a8w8_tc2_bn256"), (300, 272, 512, "a8w8_tc2h_bn256"),
                                       (2100, 4864, 1024, "a8w8_tc2h_bn256")])
def test_integer_valued_bit_exact(M, N, K, cfg):
    """Integer e4m3 values |v| <= 4 and power-of-two scales: every partial sum is exact,
    so the bf16 output must equal bf16(exact) bit for bit."""
    rng = np.random.default_rng(M + N)
    codes = np.array([0x00, 0x38, 0x40, 0x44, 0x48], dtype=np.uint8)  # 0, 1, 2, 3, 4
    A_q = codes[rng.integers(0, 5, (M, K))] | (rng.integers(0, 2, (M, K)) << 7).astype(np.uint8)
    W_q = codes[rng.integers(0, 5, (N, K))] | (rng.integers(0, 2, (N, K)) << 7).astype(np.uint8)
    a_s = np.ldexp(1.0, rng.integers(-6, 3, (M, K // 128))).astype(np.float32)
    w_s = np.ldexp(1.0, rng.integers(-6, 3, ((N + 127) // 128, K // 128))).astype(np.float32)
    y = _run(A_q, a_s, W_q, w_s, cfg)
    _, ref_bf16 = ogemm.gemm_a8w8_blockscale(A_q, a_s, W_q, w_s)
    assert np.array_equal(y.float().cpu().numpy().astype(np.float64), ref_bf16)


@pytest.mark.parametrize("M,N,K", [(1, 5120, 6144), (9, 2048, 1024), (700, 1024, 1024), (2100, 5120, 1024),
                                   (4100, 9728, 1024)])
def test_deterministic_and_graph_replay(M, N, K):
    case = _raw_case(M, N, K, seed=3)
    A, a_s, W, w_s = (codes_to_device(case[0]), torch.from_numpy(case[1]).cuda(), codes_to_device(case[2]),
                      torch.from_numpy(case[3]).cuda())
    y1 = fb.gemm_a8w8_blockscale(A, a_s, W, w_s)
    y2 = fb.gemm_a8w8_blockscale(A, a_s, W, w_s)
    out = torch.empty_like(y1)
    ws = torch.zeros(max(fb.workspace_bytes(OP, M, N, K), 256), dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        fb.gemm_a8w8_blockscale(A, a_s, W, w_s, out=out, workspace=ws)
    for _ in range(3):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert np.array_equal(bf16_bits(out), bf16_bits(y1))
    assert np.array_equal(bf16_bits(y1), bf16_bits(y2))
    check_a8w8(y1, *case)


def test_m1_n5120_k6144_end_to_end():
    """M=1, N=5120, K=6144, seed 0: bf16 activations and float32 weights quantised on the
    GPU, then the GEMM; the oracle quantises and multiplies on its own."""
    x, w = inputs.m1_n5120_k6144(0)
    q, s = fb.quant_act_per_token_group(x.cuda())
    wq, ws = fb.quant_weight_block128(w.cuda())
    y = fb.gemm_a8w8_blockscale(q, s, wq, ws)
    torch.cuda.synchronize()
    A_q, a_s = oquant.quant_act_per_token_group(x.float().numpy())
    W_q, w_s = oquant.quant_weight_block128(w.numpy())
    rl, rl_bf16 = check_a8w8(y, A_q, a_s, W_q, w_s)
    assert rl < 2.2e-3  # the bf16 output-rounding floor the pages report is 1.7e-3


@pytest.mark.parametrize("nk_index", [0, 1, 2, 3])
def test_decode_sweep_full_size(nk_index):
    N, K = inputs.DECODE_NK[nk_index]
    w = inputs.weight_f32(N, K, inputs.decode_seed_w(nk_index))
    wq, ws = fb.quant_weight_block128(w.cuda())
    W_q, w_s = oquant.quant_weight_block128(w.numpy())
    assert np.array_equal(codes_from_device(wq), W_q)
    for mi, M in enumerate(inputs.DECODE_MS):
        x = inputs.activation_bf16(M, K, inputs.decode_seed_a(nk_index, mi))
        q, s = fb.quant_act_per_token_group(x.cuda())
        y = fb.gemm_a8w8_blockscale(q, s, wq, ws)
        torch.cuda.synchronize()
        A_q, a_s = oquant.quant_act_per_token_group(x.float().numpy())
        check_a8w8(y, A_q, a_s, W_q, w_s)


_PREFILL_W = {}


def _prefill_weight(nk_index):
    """Quantised prefill weight: GPU codes and scales, and the oracle's own quantisation."""
    if nk_index not in _PREFILL_W:
        _PREFILL_W.clear()  # one (N, K) at a time: 34816 x 5120 in float64 is 1.4 GB
        N, K = inputs.PREFILL_NK[nk_index]
        w = inputs.weight_f32(N, K, 11 + nk_index)
        wq, ws = fb.quant_weight_block128(w.cuda())
        W_q, w_s = oquant.quant_weight_block128(w.numpy())
        _PREFILL_W[nk_index] = (wq, ws, W_q, w_s)
    return _PREFILL_W[nk_index]


def prefill_rows(M, seed, count=256):
    """The first and last rows, every row of the last 128-row tile (the M tail when
    M % 128 != 0), the rows on both sides of a few tile boundaries, and seeded random rows
    up to `count`."""
    rng = np.random.default_rng(seed)
    last_tile = ((M - 1) // 128) * 128
    fixed = set(range(0, 8)) | set(range(last_tile, M)) | {M - 1}
    for t in rng.choice(max(1, M // 128), min(8, max(1, M // 128)), replace=False):
        fixed |= {int(t) * 128 - 1, int(t) * 128} if t > 0 else {0}
    fixed = {r for r in fixed if 0 <= r < M}
    rest = np.setdiff1d(np.arange(M), np.fromiter(fixed, dtype=np.int64))
    extra = rng.choice(rest, max(0, min(count - len(fixed), rest.size)), replace=False) if rest.size else []
    return np.unique(np.concatenate([np.fromiter(fixed, dtype=np.int64), np.asarray(extra, dtype=np.int64)]))


@pytest.mark.parametrize("M", inputs.PREFILL_MS)
@pytest.mark.parametrize("nk_index", [0, 1])
def test_prefill_full_size_sampled_rows(M, nk_index):
    """Prefill shapes at full size (1% outlier channels x20), checked on 256 rows against the
    oracle: first and last rows, the last 128-row tile, tile-boundary rows, random rows."""
    N, K = inputs.PREFILL_NK[nk_index]
    wq, ws, W_q, w_s = _prefill_weight(nk_index)
    x = inputs.activation_bf16(M, K, 12 + M + nk_index, outliers=True)
    q, s = fb.quant_act_per_token_group(x.cuda())
    y = fb.gemm_a8w8_blockscale(q, s, wq, ws)
    torch.cuda.synchronize()
    assert fb.get_device_status() == 0
    rows = prefill_rows(M, seed=M + nk_index)
    assert rows.size == 256
    A_q, a_s = oquant.quant_act_per_token_group(x.float().numpy()[rows])
    assert np.array_equal(codes_from_device(q)[rows], A_q)
    check_a8w8(y.cpu()[torch.from_numpy(rows)], A_q, a_s, W_q, w_s)


def test_prefill_m2048_n14336_full_matrix():
    """Every output of the M = 2048, N = 14336, K = 5120 prefill call against the oracle
    (checked 256 rows at a time)."""
    M = 2048
    N, K = inputs.PREFILL_NK[0]
    wq, ws, W_q, w_s = _prefill_weight(0)
    x = inputs.activation_bf16(M, K, 12 + M, outliers=True)
    q, s = fb.quant_act_per_token_group(x.cuda())
    y = fb.gemm_a8w8_blockscale(q, s, wq, ws)
    torch.cuda.synchronize()
    assert fb.get_device_status() == 0
    A_q, a_s = oquant.quant_act_per_token_group(x.float().numpy())
    yc = y.cpu()
    for r0 in range(0, M, 256):
        check_a8w8(yc[r0:r0 + 256], A_q[r0:r0 + 256], a_s[r0:r0 + 256], W_q, w_s)


def test_ladder_every_tile_tail_class():
    """The dense-M ladder on (5120, 6144): one M from every residue class mod 128 in
    257..8192 (seeded), each checked on its last 128-row tile -- the M-tail rows -- and
    its first rows. The activations of all calls are row prefixes of one quantised
    8192 x 6144 matrix."""
    N, K = inputs.LADDER_NK
    w = inputs.weight_f32(N, K, 31)
    wq, ws = fb.quant_weight_block128(w.cuda())
    W_q, w_s = oquant.quant_weight_block128(w.numpy())
    x = inputs.activation_bf16(8192, K, 32)
    q, s = fb.quant_act_per_token_group(x.cuda())
    rng = np.random.default_rng(33)
    ms = sorted(257 + r + 128 * int(rng.integers(0, (8192 - 257 - r) // 128 + 1)) for r in range(128))
    assert len({m % 128 for m in ms}) == 128 and max(ms) <= 8192
    rows_of = {M: np.concatenate([np.arange(0, 2), np.arange(((M - 1) // 128) * 128, M)]) for M in ms}
    ys = {}
    for M in ms:
        y = fb.gemm_a8w8_blockscale(q[:M], s[:M], wq, ws)
        ys[M] = y[torch.from_numpy(rows_of[M]).cuda()].cpu()
    torch.cuda.synchronize()
    assert fb.get_device_status() == 0
    xf = x.float().numpy()
    for M in ms:
        A_q, a_s = oquant.quant_act_per_token_group(xf[rows_of[M]])
        check_a8w8(ys[M], A_q, a_s, W_q, w_s)


def test_workspace_shared_across_shapes():
    """Calls of different shapes and kernels share one workspace in stream order (every
    call leaves its arrival counters at zero)."""
    shapes = [(1, 5120, 6144), (16, 34816, 5120), (9, 2048, 1024), (3, 14336, 5120), (1, 5120, 6144)]
    need = max(fb.workspace_bytes(OP, *s) for s in shapes)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    for i, (M, N, K) in enumerate(shapes):
        case = _raw_case(M, N, K, seed=100 + i)
        y = fb.gemm_a8w8_blockscale(codes_to_device(case[0]), torch.from_numpy(case[1]).cuda(),
                                    codes_to_device(case[2]), torch.from_numpy(case[3]).cuda(), workspace=ws)
        torch.cuda.synchronize()
        check_a8w8(y, *case)
    # the same sequence again on the now-used workspace: bit-identical outputs
    for cfg in ("a8w8_gemv_d4", "a8w8_gemv_tma", "a8w8_gemv_umma"):
        fb.dispatch_set_row(OP, 9, 2048, 1024, cfg)
        try:
            case = _raw_case(9, 2048, 1024, seed=102)
            args = (codes_to_device(case[0]), torch.from_numpy(case[1]).cuda(), codes_to_device(case[2]),
                    torch.from_numpy(case[3]).cuda())
            y1 = fb.gemm_a8w8_blockscale(*args, workspace=ws)
            y2 = fb.gemm_a8w8_blockscale(*args, workspace=ws)
            torch.cuda.synchronize()
            assert np.array_equal(bf16_bits(y1), bf16_bits(y2))
            check_a8w8(y1, *case)
        finally:
            fb.dispatch_reset_table(True)


@pytest.mark.parametrize("M,N,K", [(1, 5120, 6144), (16, 34816, 5120), (9, 2048, 1024), (3, 144, 384)])
def test_static_weights_flag_bit_identical(M, N, K):
    """FP8BS_FLAG_STATIC_WEIGHTS only moves the weight fetch earlier: same bits, also when
    the call follows a kernel that writes its activations (the quantiser) in one graph."""
    case = _raw_case(M, N, K, seed=7 + M)
    A, a_s, W, w_s = (codes_to_device(case[0]), torch.from_numpy(case[1]).cuda(), codes_to_device(case[2]),
                      torch.from_numpy(case[3]).cuda())
    ref = fb.gemm_a8w8_blockscale(A, a_s, W, w_s)
    y = fb.gemm_a8w8_blockscale(A, a_s, W, w_s, static_weights=True)
    torch.cuda.synchronize()
    assert np.array_equal(bf16_bits(y), bf16_bits(ref))
    # quantiser -> GEMM chains in one graph, the GEMM reading what the quantiser wrote
    x = inputs.activation_bf16(M, K, seed=M)
    xd = x.cuda()
    q = torch.empty((M, K), dtype=torch.float8_e4m3fn, device="cuda")
    s = torch.empty((M, K // 128), dtype=torch.float32, device="cuda")
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(max(fb.workspace_bytes(OP, M, N, K), 256), dtype=torch.uint8, device="cuda")
    st = torch.cuda.Stream()
    st.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=st):
        for _ in range(3):
            fb.quant_act_per_token_group(xd, q=q, scale=s, stream=st)
            fb.gemm_a8w8_blockscale(q, s, W, w_s, out=out, workspace=ws, stream=st, static_weights=True)
    g.replay()
    torch.cuda.synchronize()
    q2, s2 = fb.quant_act_per_token_group(xd)
    ref2 = fb.gemm_a8w8_blockscale(q2, s2, W, w_s)
    torch.cuda.synchronize()
    assert np.array_equal(bf16_bits(out), bf16_bits(ref2))
