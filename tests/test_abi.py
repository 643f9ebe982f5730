"""The C ABI library: loads, exports every symbol include/fp8bs.h declares, validates
arguments and runs its host-side dispatch logic -- all without a GPU (no compute call
reaches a kernel here: each either fails validation or is host-only)."""

import ctypes
import os
import re
import subprocess

import pytest

import fp8_block_scaled_a8w8_b200 as fb
from oracle import dispatch as odispatch
from fp8_block_scaled_a8w8_b200 import inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    from fp8_block_scaled_a8w8_b200 import build
    build.build()
    yield


def _declared():
    src = open(os.path.join(ROOT, "include", "fp8bs.h")).read()
    return sorted(set(re.findall(r"\b(fp8bs_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol():
    decl = _declared()
    assert len(decl) >= 16
    out = subprocess.run(["nm", "-D", "--defined-only", fb.LIB_PATH], capture_output=True, text=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if l.strip()}
    missing = [d for d in decl if d not in exported]
    assert not missing, missing
    l = fb.lib()
    for d in decl:
        assert getattr(l, d) is not None


def test_version_and_status_strings():
    assert "sm_100a" in fb.version()
    for code in range(7):
        assert fb.status_string(code)


def test_argument_validation_without_gpu():
    l = fb.lib()
    P = 0x10000  # never dereferenced: validation fails first
    # null pointers
    assert l.fp8bs_gemm_a8w8_blockscale(None, P, P, P, P, 1, 128, 128, None, 0, None) == 1
    # K % 128, N % 16, non-positive sizes
    assert l.fp8bs_gemm_a8w8_blockscale(P, P, P, P, P, 1, 128, 100, None, 0, None) == 1
    assert l.fp8bs_gemm_a8w8_blockscale(P, P, P, P, P, 1, 120, 128, None, 0, None) == 1
    assert l.fp8bs_gemm_a8w8_blockscale(P, P, P, P, P, 0, 128, 128, None, 0, None) == 1
    # misaligned pointer
    assert l.fp8bs_gemm_a8w8_blockscale(P + 1, P, P, P, P, 1, 128, 128, None, 0, None) == 3
    assert l.fp8bs_gemm_bf16(P, P + 8, P, 0, 4, 32, 64, None, 0, None) == 3
    # tiled weights: sizes, tiling arguments, unknown GEMM flag bits
    assert fb.tiled_weight_bytes(5120, 6144) == 40 * 48 * 16384
    assert fb.tiled_weight_bytes(400, 1408) == 4 * 11 * 16384  # block count rounded up to even
    assert fb.tiled_weight_bytes(128, 100) == 0
    assert l.fp8bs_tile_weight_e4m3(None, 128, 128, P, None) == 1
    assert l.fp8bs_tile_weight_e4m3(P, 128, 100, P, None) == 1
    assert l.fp8bs_tile_weight_e4m3(P, 128, 128, P + 4, None) == 3
    assert l.fp8bs_gemm_a8w8_blockscale_ex(P, P, P, P, P, 1, 128, 128, None, 0, 4, None) == 1
    assert l.fp8bs_gemm_bf16(P, P, P, 0, 4, 32, 96, None, 0, None) == 1
    # quantisers: group must be 128, ld_x >= K and a multiple of 8
    assert l.fp8bs_quant_act_per_token_group(P, 2, 256, 256, P, P, 64, None) == 1
    assert l.fp8bs_quant_act_per_token_group(P, 2, 256, 128, P, P, 128, None) == 1
    assert l.fp8bs_quant_act_per_token_group(P, 2, 256, 260, P, P, 128, None) == 3
    assert l.fp8bs_quant_weight_block128(P, 100, 200, P, P, None) == 1


def test_c_dispatch_walk_matches_page_examples(golden_dir):
    try:
        for line in open(os.path.join(golden_dir, "padded_m_examples.txt")):
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            table, m, want = [t.strip() for t in line.split(";")]
            fb.dispatch_reset_table(keep_builtin=False)
            for r in table.split(","):
                fb.dispatch_set_row(fb.OP_A8W8_BLOCKSCALE, int(r), 5120, 6144, "a8w8_tc_bn256")
            pm, cfg = fb.dispatch_lookup(fb.OP_A8W8_BLOCKSCALE, int(m), 5120, 6144)
            assert pm == (None if want == "miss" else int(want)), (table, m, want, pm)
            if pm is None:  # a miss runs the shape's default configuration
                assert cfg == ("a8w8_gemv_umma" if int(m) <= 32 else "a8w8_tcw_bn256")
    finally:
        fb.dispatch_reset_table(keep_builtin=True)


def test_c_dispatch_walk_matches_oracle_on_ladder():
    rows = {1, 2, 4, 8, 24, 48, 64, 96, 128, 512, 2048, 8192}
    try:
        fb.dispatch_reset_table(keep_builtin=False)
        for r in rows:
            fb.dispatch_set_row(fb.OP_BF16, r, 256, 6144, "bf16_tc_bn256" if r > 32 else "bf16_gemv_d4")
        for m in list(range(1, 300)) + inputs.ladder_ms():
            pm, _ = fb.dispatch_lookup(fb.OP_BF16, m, 256, 6144)
            assert pm == odispatch.lookup(rows, m), m
    finally:
        fb.dispatch_reset_table(keep_builtin=True)


def test_census_counts_and_dedup():
    fb.dispatch_reset_stats()
    for _ in range(3):
        fb.dispatch_lookup(fb.OP_A8W8_BLOCKSCALE, 3, 5120, 6144, record=True)  # built-in row 4
    fb.dispatch_lookup(fb.OP_A8W8_BLOCKSCALE, 6016, 14336, 5120, record=True)  # -> 8192 row
    fb.dispatch_lookup(fb.OP_A8W8_BLOCKSCALE, 40, 1024, 1024, record=True)     # no row: miss
    fb.dispatch_lookup(fb.OP_A8W8_BLOCKSCALE, 40, 1024, 1024, record=False)    # not counted
    st = fb.dispatch_stats(fb.OP_A8W8_BLOCKSCALE)
    assert st == {"hits": 4, "misses": 1, "distinct_hits": 2, "distinct_misses": 1}
    recs = fb.dispatch_dump_json()
    by_m = {r["M"]: r for r in recs}
    assert by_m[3]["padded_M"] == 4 and by_m[3]["count"] == 3 and by_m[3]["hit"]
    assert by_m[6016]["padded_M"] == 8192
    # a miss runs the default: 1 x 4 tiles of 256 columns would leave most SMs idle, so 128
    assert by_m[40]["hit"] is False and by_m[40]["cfg"] == "a8w8_tcw_bn128"
    fb.dispatch_reset_stats()
    assert fb.dispatch_stats(fb.OP_A8W8_BLOCKSCALE)["hits"] == 0


def test_table_hash_tracks_rows():
    h0 = fb.dispatch_table_hash()
    try:
        fb.dispatch_set_row(fb.OP_A8W8_BLOCKSCALE, 4, 5120, 6144, "a8w8_gemv_d2")
        assert fb.dispatch_table_hash() != h0
    finally:
        fb.dispatch_reset_table(keep_builtin=True)
    assert fb.dispatch_table_hash() == h0


def test_set_row_rejects_unknown_and_gemv_for_large_m():
    with pytest.raises(fb.Fp8bsError):
        fb.dispatch_set_row(fb.OP_A8W8_BLOCKSCALE, 4, 5120, 6144, "no_such_kernel")
    with pytest.raises(fb.Fp8bsError):
        fb.dispatch_set_row(fb.OP_A8W8_BLOCKSCALE, 64, 5120, 6144, "a8w8_gemv_d4")
    assert "a8w8_tc_bn256" in fb.dispatch_list_configs(fb.OP_A8W8_BLOCKSCALE)
    assert "bf16_tc_bn32" in fb.dispatch_list_configs(fb.OP_BF16)


def test_product_package_does_not_import_oracle():
    pkg = os.path.join(ROOT, "fp8_block_scaled_a8w8_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".cpp", ".h")):
                src = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(from|import)\s+oracle\b", src, re.M), f
                assert "oracle/" not in src, f
