"""The dispatch table's measured rows (csrc/tuned_rows.inc, written by the package's
tune.py): every row is in the table with its measured configuration and marked tuned, and
the census can tell a tuned hit from the default heuristic because some rows name another
configuration than a miss would run ([aiter#7752] "Details": the dispatch reads the
kernel name; [cookbook#8]: a hit on a tuned row is only worth counting if the row differs
from what a miss runs)."""

import os
import re

import fp8_block_scaled_a8w8_b200 as fb

INC = os.path.join(os.path.dirname(fb.__file__), "csrc", "tuned_rows.inc")
ROW = re.compile(r'^\{(\d+), (\d+), (\d+), (\d+), "([a-z0-9_]+)"\},$')


def _rows():
    out = []
    for line in open(INC):
        m = ROW.match(line.strip())
        if m:
            out.append((int(m.group(1)), int(m.group(2)), int(m.group(3)), int(m.group(4)), m.group(5)))
    return out


def _defaults(keys):
    fb.dispatch_reset_table(keep_builtin=False)
    try:
        return {k: fb.dispatch_lookup(*k)[1] for k in keys}
    finally:
        fb.dispatch_reset_table(keep_builtin=True)


def test_tuned_rows_are_in_the_table():
    rows = _rows()
    assert rows, "no measured rows"
    fb.dispatch_reset_table(keep_builtin=True)
    table = {(r["op"], r["M"], r["N"], r["K"]): r for r in fb.dispatch_dump_table()}
    for op, M, N, K, cfg in rows:
        assert cfg in fb.dispatch_list_configs(op)
        pm, got = fb.dispatch_lookup(op, M, N, K)
        assert pm == M and got == cfg, (op, M, N, K, cfg, got)
        assert table[(op, M, N, K)]["tuned"] and table[(op, M, N, K)]["cfg"] == cfg


def test_some_tuned_rows_differ_from_the_default():
    rows = _rows()
    dflt = _defaults([(op, M, N, K) for op, M, N, K, _ in rows])
    differ = [(k, cfg) for *k, cfg in rows if dflt[tuple(k)] != cfg]
    assert differ, "every measured row equals the default heuristic"
    # one pinned example: M = 64 on the (5120, 6144) projection, where the measured choice
    # is not the wide-epilogue default
    k = (fb.OP_A8W8_BLOCKSCALE, 64, 5120, 6144)
    cfg = dict(((op, M, N, K), c) for op, M, N, K, c in rows).get(k)
    if cfg is not None:
        assert fb.dispatch_lookup(*k)[1] == cfg


def test_set_row_clears_the_tuned_mark():
    op, M, N, K, cfg = _rows()[0]
    try:
        fb.dispatch_set_row(op, M, N, K, cfg)
        row = [r for r in fb.dispatch_dump_table() if (r["op"], r["M"], r["N"], r["K"]) == (op, M, N, K)][0]
        assert not row["tuned"]
    finally:
        fb.dispatch_reset_table(keep_builtin=True)
    row = [r for r in fb.dispatch_dump_table() if (r["op"], r["M"], r["N"], r["K"]) == (op, M, N, K)][0]
    assert row["tuned"]
