"""Dispatch-table tuner: times every applicable kernel configuration on each built-in table
row and writes the measured choice into csrc/tuned_rows.inc (compiled into the library).

    python -m fp8_block_scaled_a8w8_b200.tune [--out PATH] [--ops 0,1] [--rounds 5]

The table's rows are the (op, M, N, K) keys the padded-M walk lands on ([aiter#7752]
"Retune gfx942 ... a8w8 blockscale decode rows for cold weights": rows are tuned with
weights read cold from HBM, as a decode step reads them; the dispatch reads only the
kernel name and split, "Details"). Every configuration is timed on the row's exact shape:
R back-to-back calls captured in one CUDA graph, weights rotated over copies that exceed
the L2, the median of interleaved rounds. The fastest wins, unless the per-shape default
is within the noise margin of it (then the default is kept, so that a row only departs from
the heuristic on a measured difference). A row the tuner times is marked tuned in the
table (fp8bs_dispatch_dump_table_json).
"""

from __future__ import annotations

import argparse
import os
import sys
import time

import torch

import fp8_block_scaled_a8w8_b200 as fb

HERE = os.path.dirname(os.path.abspath(__file__))
DEFAULT_OUT = os.path.join(HERE, "csrc", "tuned_rows.inc")
ROTATE_BYTES = 384 << 20  # weight copies per shape: > 3x the 126 MB L2
MARGIN = 0.015            # keep the default unless a candidate is > 1.5% faster


def candidates(op: int, M: int, N: int) -> list:
    names = fb.dispatch_list_configs(op)
    small = M <= 32
    out = []
    for c in names:
        gemv = "_gemv" in c
        if gemv != small:
            continue
        if "_sk" in c and M > 512:  # fixed splits: only where the tiles leave SMs idle
            continue
        if op == fb.OP_BF16 and not small:
            bn = int(c.rsplit("bn", 1)[1])
            if bn > N and N % 32 == 0 and bn != 32:
                continue
        out.append(c)
    return out


def default_configs(rows) -> dict:
    """The configuration a miss runs (the per-shape heuristic) for each row key."""
    fb.dispatch_reset_table(keep_builtin=False)
    try:
        return {(r["op"], r["M"], r["N"], r["K"]): fb.dispatch_lookup(r["op"], r["M"], r["N"], r["K"])[1] for r in rows}
    finally:
        fb.dispatch_reset_table(keep_builtin=True)


def _operands(op, M, N, K, dev):
    g = torch.Generator(device=dev).manual_seed(M * 7919 + N * 31 + K)
    if op == fb.OP_A8W8_BLOCKSCALE:
        x = (torch.randn(M, K, device=dev, generator=g)).to(torch.bfloat16)
        q, s = fb.quant_act_per_token_group(x)
        copies = max(1, min(16, -(-ROTATE_BYTES // (N * K))))
        ws = []
        for _ in range(copies):
            w = torch.randn(N, K, device=dev, generator=g) * 0.02
            ws.append(fb.quant_weight_block128(w))
        out = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        return (q, s), ws, out
    x = (torch.randn(M, K, device=dev, generator=g)).to(torch.bfloat16)
    copies = max(1, min(16, -(-ROTATE_BYTES // (2 * N * K))))
    ws = [(torch.randn(N, K, device=dev, generator=g) * 0.02).to(torch.bfloat16) for _ in range(copies)]
    out = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    return (x,), ws, out


def _call(op, a, w, out, workspace, stream):
    if op == fb.OP_A8W8_BLOCKSCALE:
        fb.gemm_a8w8_blockscale(a[0], a[1], w[0], w[1], out=out, workspace=workspace, stream=stream,
                                static_weights=True)
    else:
        fb.gemm_bf16(a[0], w, out=out, workspace=workspace, stream=stream)


def time_row(op, M, N, K, cands, rounds, R, dev, stream):
    """Median us/call of each candidate (None where the configuration rejects the shape)."""
    need = 1
    for c in cands:
        fb.dispatch_set_row(op, M, N, K, c)
        need = max(need, fb.workspace_bytes(op, M, N, K))
    workspace = torch.zeros(need, dtype=torch.uint8, device=dev)
    a, ws, out = _operands(op, M, N, K, dev)
    graphs = {}
    for c in cands:
        fb.dispatch_set_row(op, M, N, K, c)
        try:
            with torch.cuda.stream(stream):
                for i in range(2):  # warm-up (also surfaces a rejected shape)
                    _call(op, a, ws[i % len(ws)], out, workspace, stream)
                stream.synchronize()
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    for r in range(R):
                        _call(op, a, ws[r % len(ws)], out, workspace, stream)
            graphs[c] = g
        except fb.Fp8bsError:
            graphs[c] = None
        # a graph captures the kernel choice: the row may change for the next candidate
    times = {c: [] for c in cands}
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(rounds):
        for c, g in graphs.items():
            if g is None:
                continue
            with torch.cuda.stream(stream):
                e0.record(stream)
                g.replay()
                e1.record(stream)
            e1.synchronize()
            times[c].append(e0.elapsed_time(e1) * 1000.0 / R)
    if fb.get_device_status(stream) != 0:
        raise RuntimeError(f"device status set while timing op={op} M={M} N={N} K={K}")
    graphs.clear()
    return {c: (sorted(t)[len(t) // 2] if t else None) for c, t in times.items()}


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--out", default=DEFAULT_OUT)
    ap.add_argument("--ops", default="0,1")
    ap.add_argument("--rounds", type=int, default=5)
    ap.add_argument("--calls", type=int, default=8)
    a = ap.parse_args(argv)
    assert torch.cuda.is_available(), "the tuner times kernels on a GPU"
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    ops = [int(x) for x in a.ops.split(",")]
    fb.dispatch_reset_table(keep_builtin=True)
    table = [r for r in fb.dispatch_dump_table() if r["op"] in ops]
    defaults = default_configs(table)
    stream = torch.cuda.Stream(device=dev)
    prop = torch.cuda.get_device_properties(dev)
    lines = [f"// Generated by fp8_block_scaled_a8w8_b200/tune.py on {prop.name} ({prop.multi_processor_count} SMs), "
             f"{time.strftime('%Y-%m-%d')}.",
             "// Each row: the fastest configuration timed on the row's shape (us/call, cold weights, CUDA graph of",
             f"// {a.calls} calls, median of {a.rounds} rounds); the default is kept unless beaten by > {MARGIN:.1%}.",
             "// {op, M, N, K, configuration}"]
    changed = 0
    t_start = time.time()
    for r in table:
        op, M, N, K = r["op"], r["M"], r["N"], r["K"]
        dflt = defaults[(op, M, N, K)]
        cands = candidates(op, M, N)
        if dflt not in cands:
            cands.append(dflt)
        us = time_row(op, M, N, K, cands, a.rounds, a.calls, dev, stream)
        ok = {c: t for c, t in us.items() if t is not None}
        best = min(ok, key=ok.get)
        choice = dflt if (dflt in ok and ok[dflt] <= ok[best] * (1 + MARGIN)) else best
        changed += choice != dflt
        detail = " ".join(f"{c}={t:.2f}" for c, t in sorted(ok.items(), key=lambda kv: kv[1]))
        lines.append(f"// op={op} M={M} N={N} K={K} default={dflt}: {detail}")
        lines.append(f"{{{op}, {M}, {N}, {K}, \"{choice}\"}},")
        print(f"op={op} M={M:5d} N={N:5d} K={K:5d}: {choice:18s} (default {dflt}) {detail}", flush=True)
    fb.dispatch_reset_table(keep_builtin=True)
    with open(a.out, "w") as f:
        f.write("\n".join(lines) + "\n")
    print(f"{len(table)} rows timed in {time.time() - t_start:.0f} s, {changed} differ from the default; wrote {a.out}")
    return 0


if __name__ == "__main__":
    sys.exit(main())
