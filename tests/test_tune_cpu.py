"""The tuner's host logic (no GPU): which configurations it times for a row, and that every
committed row names a configuration the tuner could have chosen for that shape (a timed
candidate, or the shape's default, which is always timed)."""

import os
import re

import fp8_block_scaled_a8w8_b200 as fb
from fp8_block_scaled_a8w8_b200 import tune

INC = os.path.join(os.path.dirname(fb.__file__), "csrc", "tuned_rows.inc")
ROW = re.compile(r'^\{(\d+), (\d+), (\d+), (\d+), "([a-z0-9_]+)"\},$')
A8, BF = fb.OP_A8W8_BLOCKSCALE, fb.OP_BF16


def test_decode_rows_time_only_weight_streaming_kernels():
    c = tune.candidates(A8, 16, 5120)
    assert c and all("_gemv" in n for n in c)
    assert "a8w8_gemv_umma" in c and "a8w8_gemv_tma" in c


def test_mid_m_rows_time_tiled_kernels_and_fixed_splits():
    c = tune.candidates(A8, 48, 5120)
    assert not any("_gemv" in n for n in c)
    assert {"a8w8_tcw_bn256", "a8w8_tc_bn256", "a8w8_tcw_bn128_sk8", "a8w8_tc2_bn256"} <= set(c)


def test_large_m_rows_skip_fixed_splits():
    c = tune.candidates(A8, 1024, 5120)
    assert c and not any("_sk" in n for n in c)
    assert "a8w8_tcw_bn256" in c


def test_bf16_rows_skip_tiles_wider_than_n():
    assert tune.candidates(BF, 576, 32) == ["bf16_tc_bn32"]
    c = tune.candidates(BF, 576, 128)
    assert "bf16_tc_bn192" not in c and "bf16_tc_bn256" not in c and "bf16_tc_bn128" in c
    assert "bf16_tc_bn256" in tune.candidates(BF, 576, 32320)


def test_committed_rows_are_tuner_choices():
    rows = []
    for line in open(INC):
        m = ROW.match(line.strip())
        if m:
            rows.append((int(m.group(1)), int(m.group(2)), int(m.group(3)), int(m.group(4)), m.group(5)))
    assert len(rows) >= 100
    dflt = tune.default_configs([{"op": op, "M": M, "N": N, "K": K} for op, M, N, K, _ in rows])
    for op, M, N, K, cfg in rows:
        assert cfg in tune.candidates(op, M, N) or cfg == dflt[(op, M, N, K)], (op, M, N, K, cfg)
