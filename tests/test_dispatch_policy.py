"""Default kernel choice and workspace sizing (host logic, no GPU).

Restates the documented policy in Python and checks the library's choices against it:
M <= 32 runs the weight-streaming kernel; otherwise the tiled kernel takes the widest tile
whose output tiles give at least half of the SMs a tile, and splits K (workspace > 0)
only when even the narrowest tile leaves that many SMs idle, into as many splits as keep
the tiles x splits work items within one wave of SMs. Without a
GPU the library assumes 148 SMs (B200).
"""

import math

import pytest

import fp8_block_scaled_a8w8_b200 as fb

SMS = 148
KCOUNTER = 65536 * 4


def _pick(M, N, cands):
    m_tiles = math.ceil(M / 128)
    for b in cands:
        if m_tiles * math.ceil(N / b) >= (SMS + 1) // 2:
            return b
    return cands[-1]


def _splits(M, N, K, bn, kb):
    tiles = math.ceil(M / 128) * math.ceil(N / bn)
    if 2 * tiles >= SMS:
        return 1
    return max(1, min(SMS // tiles, kb // 2, 8, kb))  # one wave: tiles x splits <= SMs


@pytest.mark.parametrize("M", [33, 64, 100, 128, 256, 300, 565, 1099, 2048, 8192])
@pytest.mark.parametrize("N,K", [(5120, 6144), (14336, 5120), (1024, 1024), (384, 640)])
def test_a8w8_tiled_choice(M, N, K):
    bn = _pick(M, N, [256, 128]) if N % 256 == 0 else 128
    fb.dispatch_reset_table(keep_builtin=False)  # no table rows: every lookup runs the default
    try:
        _, cfg = fb.dispatch_lookup(fb.OP_A8W8_BLOCKSCALE, M, N, K)
        assert cfg == f"a8w8_tcw_bn{bn}"
        sp = _splits(M, N, K, bn, K // 128)
        ws = fb.workspace_bytes(fb.OP_A8W8_BLOCKSCALE, M, N, K)
        tiles = math.ceil(M / 128) * math.ceil(N / bn)
        assert ws == (0 if sp == 1 else KCOUNTER + tiles * sp * 128 * bn * 4)
    finally:
        fb.dispatch_reset_table(keep_builtin=True)


@pytest.mark.parametrize("M", [576, 4096, 16384, 40, 200, 24 + 16, 3072])
@pytest.mark.parametrize("N,K", [(256, 6144), (32, 6144), (384, 5120), (1024, 5120), (128, 512), (48, 192),
                                 (32320, 5120), (2064, 1024)])
def test_bf16_tiled_choice(M, N, K):
    if N >= 2048:  # large N: 256 or 128 even with a ragged last tile
        cands = [256, 128]
    else:
        cands = [b for b in (256, 192, 128, 64, 32) if b <= N and N % b == 0] or [32]
    if N < 256 and N % 32 == 0 and N != cands[0]:
        cands = [N] + cands
    bn = _pick(M, N, cands)
    if bn not in (32, 64, 128, 192, 256):
        bn = 32
    fb.dispatch_reset_table(keep_builtin=False)
    try:
        _, cfg = fb.dispatch_lookup(fb.OP_BF16, M, N, K)
        assert cfg == f"bf16_tc_bn{bn}"
        sp = _splits(M, N, K, bn, K // 64)
        tiles = math.ceil(M / 128) * math.ceil(N / bn)
        assert fb.workspace_bytes(fb.OP_BF16, M, N, K) == (0 if sp == 1 else KCOUNTER + tiles * sp * 128 * bn * 4)
    finally:
        fb.dispatch_reset_table(keep_builtin=True)


@pytest.mark.parametrize("M", [1, 2, 3, 8, 9, 16, 17, 31, 32])
def test_small_m_takes_weight_streaming(M):
    fb.dispatch_reset_table(keep_builtin=False)
    try:
        assert fb.dispatch_lookup(fb.OP_A8W8_BLOCKSCALE, M, 5120, 6144)[1] == "a8w8_gemv_umma"
        assert fb.dispatch_lookup(fb.OP_BF16, M, 256, 6144)[1] == "bf16_gemv_umma"
    finally:
        fb.dispatch_reset_table(keep_builtin=True)


@pytest.mark.parametrize("M,N,K", [(1, 5120, 6144), (16, 34816, 5120), (32, 16384, 5120), (1, 16, 128)])
def test_weight_streaming_workspace(M, N, K):
    """Counters + two fp32 partial slots of 32 token rows x 128 weight rows per CTA; the CTA
    count is min(SMs, units / 8) with units = 128-row blocks x 128-byte K chunks. The a8w8
    size also covers the mma.sync kernel it may hand over to (whose partials hold
    8 * ceil(M / 8) token columns for each of 8 warps x 16 rows)."""
    def ctas(units):
        return max(1, min(SMS, units // 8))
    nblk = math.ceil(N / 128)
    own8 = KCOUNTER + 2 * ctas(nblk * (K // 128)) * 32 * 128 * 4
    tma = KCOUNTER + 2 * min(SMS, nblk * (K // 128)) * 8 * math.ceil(M / 8) * 4 * 32 * 4
    assert fb.workspace_bytes(fb.OP_A8W8_BLOCKSCALE, M, N, K) == max(own8, tma)
    own16 = KCOUNTER + 2 * ctas(nblk * (K // 64)) * 32 * 128 * 4
    assert fb.workspace_bytes(fb.OP_BF16, M, N, K) == own16


def _mx_split(tiles, kb):
    return 1 if 2 * tiles >= SMS else max(1, min(SMS // tiles, kb // 2, 8, kb))


def _mx_bn(batch, M, N, K):
    mt = batch * math.ceil(M / 128)
    t192, t256 = mt * math.ceil(N / 192), mt * math.ceil(N / 256)
    if t192 > SMS and t256 <= SMS:
        return 256
    if batch == 1 and 2 * t192 < SMS:  # fewer K stages per CTA at 1.15 the cost per stage
        kb = K // 128
        if 115 * math.ceil(kb / _mx_split(t256, kb)) < 100 * math.ceil(kb / _mx_split(t192, kb)):
            return 256
    return 192


@pytest.mark.parametrize("batch,M,N,K", [(1, 48, 1792, 5120), (1, 768, 1792, 5120), (1, 48, 4608, 5120),
                                         (1, 768, 4608, 5120), (1, 768, 5120, 2304), (1, 768, 5120, 8192),
                                         (1, 48, 32768, 1280), (8, 16, 1024, 4096), (8, 64, 1024, 4096),
                                         (1, 1, 192, 128), (1, 40, 256, 256)])
def test_mx32_tiles_and_splits(batch, M, N, K):
    """MX32: 192-wide tiles, or 256-wide ones (one accumulator) when 192-wide tiles would
    spill into a partial second wave that 256-wide tiles avoid, or, for a single GEMM that
    splits K, when 256-wide tiles leave each CTA fewer K stages (a stage counted 1.15 times);
    K is split only when the tiles leave half the SMs idle, into as many splits as keep one
    wave, at most 8, each at least 2 K blocks (workspace = counters + one fp32 partial tile
    per split)."""
    kb = K // 128
    bn = _mx_bn(batch, M, N, K)
    tiles = batch * math.ceil(M / 128) * math.ceil(N / bn)
    sp = _mx_split(tiles, kb)
    want = 0 if sp == 1 else KCOUNTER + tiles * sp * 128 * bn * 4
    assert fb.mx32_workspace_bytes(batch, M, N, K) == want
    if (batch, M, N, K) == (1, 768, 5120, 8192):
        assert bn == 256 and sp == 1  # 162 tiles of 192 against 120 of 256 on 148 SMs
    if (batch, M, N, K) == (1, 48, 1792, 5120):
        assert bn == 192 and sp == 8
    if (batch, M, N, K) == (1, 768, 1792, 5120):
        assert bn == 256 and sp == 3  # 42 tiles x 3 splits: 14 K blocks a CTA against 20
    if batch == 8:
        assert bn == 192
