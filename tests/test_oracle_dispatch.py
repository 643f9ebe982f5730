"""Pins for the oracle's padded-M walk and census rule (CPU only)."""

import os

import pytest

from oracle import dispatch


def _examples(golden_dir):
    rows = []
    for line in open(os.path.join(golden_dir, "padded_m_examples.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        table, m, want = [t.strip() for t in line.split(";")]
        rows.append(({int(x) for x in table.split(",")}, int(m), None if want == "miss" else int(want)))
    return rows


def test_page_examples(golden_dir):
    ex = _examples(golden_dir)
    assert len(ex) >= 25
    for table, m, want in ex:
        assert dispatch.lookup(table, m) == want, (sorted(table), m, want)


def test_probe_sequence_shape():
    assert dispatch.probe_sequence(1) == [1]
    assert dispatch.probe_sequence(3) == [3, 4]
    assert dispatch.probe_sequence(16) == [16]
    assert dispatch.probe_sequence(17) == [17, 32]
    assert dispatch.probe_sequence(100) == [100, 112, 128]
    assert dispatch.probe_sequence(256) == [256]
    assert dispatch.probe_sequence(257) == [257, 512]
    assert dispatch.probe_sequence(6016) == [6016, 8192]
    with pytest.raises(ValueError):
        dispatch.probe_sequence(0)


def test_exact_row_wins_over_padding():
    assert dispatch.lookup({5, 8}, 5) == 5
    assert dispatch.lookup({24, 32}, 20) == 32  # 20 -> band 32 (next multiple of 16), not 24


def test_census_dedup_per_worker():
    """[cookbook#8] review comment 1: each TP worker logs the same lookup; count it once."""
    rec = dict(M=3, N=256, K=6144, table="bf16.csv", padded_M=4, lib="x")
    miss = dict(M=6016, N=256, K=6144, table="bf16.csv", padded_M=None, lib="x")
    recs = [dict(rec) for _ in range(8)] + [dict(miss) for _ in range(8)]
    assert dispatch.census(recs) == (1, 1, 1)
