"""Benchmark: a8w8 block-scale GEMM, us/call, TFLOPS and HBM GB/s on cold weights vs roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

Headline workload (N=1): the decode sweep -- M in {1,2,3,4,8,9,16} on the four
Qwen3.8-27B projections (N,K) = (5120,6144), (14336,5120), (16384,5120),
(34816,5120) of [aiter#7752] "Kernel". One step is one pass of the hot path over
the sweep: for each of the 28 (M,N,K) calls, per-token 1x128 activation
quantisation, dispatch, and the block-scaled GEMM. Weights are quantised once
(set-up) and rotated over >= 512 MiB of distinct device copies per shape, so every
call reads cold weights from HBM ([vllm#1065]: a 48 MiB rotation was 19%
optimistic, 512 MiB within 1.1% of in-model timing). The working set of every
step is far above the 126 MB L2, which replaces an L2 flush between steps.

Each step is captured once in a CUDA graph (one graph per rotation phase) and
replayed; CUDA events recorded inside the graphs time every GEMM launch. The
timed region is bracketed by a barrier and a device synchronise on both sides and
the step time is the max over ranks. N>1 runs N independent replicas (the path
has no exchange step).

The default run also measures, with a few steps each, every other configuration: the
prefill shapes, the dense M ladder (with the dispatch census and its padded-M drift), the
bf16 small-N GEMMs, the bf16 lm_head, the fused residual add + RMSNorm + quantisation
step and the MX32 GEMMs (dense and batched), each as an entry of "workloads" with its own
roofline; the
per-shape "detail" table gives cold- and hot-weight us/call, and the CPU leg reports the
oracle's time and the accuracy of the timed outputs against it. --only skips the extra
workloads.

--impl reference times the CPU oracle (the only other arm there is) on a
bounded sample of the same workload, on the host cores.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from fp8_block_scaled_a8w8_b200 import inputs  # noqa: E402

METRIC = "a8w8 blockscale GEMM µs/call, TFLOPS & HBM GB/s (cold weights) vs roofline"
ROTATE_BYTES = int(os.environ.get("FP8BS_ROTATE_MIB", "512")) * (1 << 20)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def measured_traffic(kernel_key, algorithmic_bytes_per_launch):
    """DRAM bytes per launch from the committed ncu capture (profiles/traffic.json), scaled
    from the captured shape to this workload by algorithmic bytes (the kernels stream their
    operands once, so traffic grows in proportion). None if the kernel source changed since
    the capture."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(kernel_key)
    if not d:
        return None
    src = os.path.join(ROOT, d["source"])
    if not os.path.exists(src) or hashlib.sha256(open(src, "rb").read()).hexdigest()[:16] != d["sha256_16"]:
        return None
    return round(d["dram_bytes"] / d["algorithmic_bytes"] * algorithmic_bytes_per_launch)


def a8w8_bytes(M, N, K):
    """Algorithmic bytes of one call: A + a_scale + W + w_scale + out."""
    G = K // 128
    return M * K + 4 * M * G + N * K + 4 * ((N + 127) // 128) * G + 2 * M * N


def max_over_ranks(value_ms, device):
    """The job's time is the slowest replica's: all-reduce MAX over the process group (any
    backend; a no-op without one)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value_ms)], device=device, dtype=torch.float64)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def bf16_bytes(M, N, K, out_fp32):
    return 2 * M * K + 2 * N * K + (4 if out_fp32 else 2) * M * N


def workload_calls(name, shape=None):
    """List of (M, N, K, nk_index, m_index, outliers) for the workload."""
    if shape:
        M, N, K = (int(v) for v in shape.split(","))
        return [(M, N, K, 0, 0, False)]
    if name == "decode_sweep":
        return [(M, N, K, i, j, False) for i, (N, K) in enumerate(inputs.DECODE_NK) for j, M in enumerate(inputs.DECODE_MS)]
    if name == "decode_m1_n5120_k6144":
        return [(1, 5120, 6144, 0, 0, False)]
    if name == "prefill":
        return [(M, N, K, i, j, True) for i, (N, K) in enumerate(inputs.PREFILL_NK) for j, M in enumerate(inputs.PREFILL_MS)]
    if name == "ladder":
        N, K = inputs.LADDER_NK
        return [(M, N, K, 0, j, False) for j, M in enumerate(inputs.ladder_ms())]
    raise SystemExit(f"unknown workload {name}")


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
        time.sleep(0.3)

    def mark(self, which):
        setattr(self, which, time.time())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = []
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(parts)
            except ValueError:
                pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        load = sorted(sm)[len(sm) // 2:] if sm else []  # upper half: samples under load
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for n, v in zip(names, r[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": float(np.median(load)) if load else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(rows)}


# --------------------------------------------------------------------------- GPU arm
def init_gpu():
    """One process per GPU: (world, rank, device); NCCL process group for N > 1."""
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, torch.device("cuda", torch.cuda.current_device())


def measure_a8w8(args, world, rank, dev, workload, shape, steps, warmup, detail, e2e_steps, cpu):
    """The JSON line of one a8w8 workload (rank 0; None elsewhere). Every rank takes the
    same collective steps."""
    import torch
    import torch.distributed as dist

    import fp8_block_scaled_a8w8_b200 as fb

    fb.lib()
    pk = peaks()
    calls = workload_calls(workload, shape)
    tiled = getattr(args, "layout", "tiled") == "tiled"
    tkw = (lambda N: {"tiled_weights": True, "N": N}) if tiled else (lambda N: {})
    if getattr(args, "config", None):  # force one kernel configuration (a table row per call shape)
        for (M, N, K, *_r) in calls:
            fb.dispatch_set_row(fb.OP_A8W8_BLOCKSCALE, M, N, K, args.config)
    uses = {}
    for (M, N, K, i, j, o) in calls:
        uses[(N, K)] = uses.get((N, K), 0) + 1

    # ---- set-up (untimed): weights quantised on the GPU, rotated copies, activations
    wcopies = {}
    for (N, K), u in uses.items():
        nk_index = [nk for (_, n, k, nk, _, _) in calls if (n, k) == (N, K)][0]
        w = inputs.weight_f32(N, K, inputs.decode_seed_w(nk_index)).to(dev)
        wq, ws = fb.quant_weight_block128(w)
        del w
        if tiled:  # the weights stored in 16 KiB tiles (set-up, like the quantisation)
            wq = fb.tile_weight(wq)
        per = wq.numel() + ws.numel() * 4
        n = max(1, math.ceil(ROTATE_BYTES / per))
        n = u * math.ceil(n / u)  # a multiple of the uses per step: every step has the same period
        copies = [(wq, ws)] + [(wq.clone(), ws.clone()) for _ in range(n - 1)]
        wcopies[(N, K)] = copies
    torch.cuda.synchronize()

    # activations: one seeded base per shape (rows = largest M of that shape), calls take row
    # slices; quantised activations and outputs likewise share one buffer per shape (calls run
    # in stream order)
    maxm = {}
    for (M, N, K, i, j, o) in calls:
        maxm[(N, K)] = max(maxm.get((N, K), 0), M)
    bx, bq, bs, bo = {}, {}, {}, {}
    for (N, K), mm in maxm.items():
        i, o = [(ci, co) for (_, n, k, ci, _, co) in calls if (n, k) == (N, K)][0]
        bx[(N, K)] = inputs.activation_bf16(mm, K, inputs.decode_seed_a(i, 0), outliers=o).to(dev)
        bq[(N, K)] = torch.empty((mm, K), dtype=torch.float8_e4m3fn, device=dev)
        bs[(N, K)] = torch.empty((mm, K // 128), dtype=torch.float32, device=dev)
        bo[(N, K)] = torch.empty((mm, N), dtype=torch.bfloat16, device=dev)
    xs = [bx[(N, K)][:M] for (M, N, K, *_r) in calls]
    qs = [bq[(N, K)][:M] for (M, N, K, *_r) in calls]
    ss = [bs[(N, K)][:M] for (M, N, K, *_r) in calls]
    outs = [bo[(N, K)][:M] for (M, N, K, *_r) in calls]
    ws_bytes = max(fb.workspace_bytes(fb.OP_A8W8_BLOCKSCALE, M, N, K) for (M, N, K, *_r) in calls)
    workspace = torch.zeros(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    cfgs = [fb.dispatch_lookup(fb.OP_A8W8_BLOCKSCALE, M, N, K)[1] for (M, N, K, *_r) in calls]

    # rotation phase: step s, call c uses copy (s * uses + rank_of_c_within_shape) % n_copies
    period = 1
    for (N, K), u in uses.items():
        n = len(wcopies[(N, K)])
        period = period * (n // u) // math.gcd(period, n // u)
    if period > 64:
        raise SystemExit(f"weight rotation needs {period} graph phases; choose a rotation with a shorter period")

    stream = torch.cuda.Stream(device=dev)
    n_calls = len(calls)

    def step_launches(s, ev=None):
        """One step: the 28 activation quantisations, then the 28 GEMMs back to back (the
        calls are independent, so the GEMMs run consecutively and programmatic dependent
        launch overlaps each one's tail with the next one's weight stream)."""
        if ev is not None:
            ev[2].record(stream)
        for c in range(n_calls):
            fb.quant_act_per_token_group(xs[c], q=qs[c], scale=ss[c], stream=stream)
        if ev is not None:
            ev[0].record(stream)
        ctr = {}
        for c, (M, N, K, *_r) in enumerate(calls):
            k = ctr.get((N, K), 0)
            ctr[(N, K)] = k + 1
            cp = wcopies[(N, K)]
            wq, wsc = cp[(s * uses[(N, K)] + k) % len(cp)]
            fb.gemm_a8w8_blockscale(qs[c], ss[c], wq, wsc, out=outs[c], workspace=workspace, stream=stream,
                                    static_weights=True, **tkw(N))
        if ev is not None:
            ev[1].record(stream)

    # events inside the graphs: around the block of GEMM launches of each phase
    events = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)] for _ in range(period)]
    graphs = []
    fb.dispatch_reset_stats()
    with torch.cuda.stream(stream):
        for ph in range(period):  # eager warm-up of each phase (also loads modules)
            step_launches(ph)
        stream.synchronize()
        for ph in range(period):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                step_launches(ph, events[ph])
            graphs.append(g)
    torch.cuda.synchronize()
    census = fb.dispatch_stats(fb.OP_A8W8_BLOCKSCALE)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    with torch.cuda.stream(stream):
        for s in range(warmup):
            graphs[s % period].replay()
    barrier()

    clocks = ClockSampler(dev.index)
    if rank == 0:
        clocks.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    barrier()
    t_start.record(stream)
    for s in range(steps):
        with torch.cuda.stream(stream):
            graphs[(warmup + s) % period].replay()
    t_end.record(stream)
    barrier()
    clk = clocks.stop() if rank == 0 else None
    step_ms = t_start.elapsed_time(t_end) / steps

    # average GEMM launch duration: the GEMM block of the last replay of every phase
    gemm_block_ms = [events[ph][0].elapsed_time(events[ph][1]) for ph in sorted(
        {(warmup + s) % period for s in range(steps)})]
    gemm_ms_per_call = float(np.mean(gemm_block_ms)) / n_calls
    quant_block_ms = float(np.mean([events[ph][2].elapsed_time(events[ph][0]) for ph in sorted(
        {(warmup + s) % period for s in range(steps)})]))

    step_ms = max_over_ranks(step_ms, dev)

    # ---- end to end through the public API: pinned host inputs in, results out, per step
    e2e = None
    e2e_steps = e2e_steps if n_calls <= 64 and max(maxm.values()) <= 64 else min(e2e_steps, 3)
    if e2e_steps > 0:
        # the step's activations travel as one pinned host buffer and its results come back
        # as one: one host->device and one device->host copy per step, as a serving loop
        # moves a step's tokens
        x_off, o_off, xo, oo = [], [], 0, 0
        for (M, N, K, *_r) in calls:
            x_off.append(xo)
            o_off.append(oo)
            xo += M * K
            oo += M * N
        hx = torch.empty(xo, dtype=torch.bfloat16).pin_memory()
        for c, x in enumerate(xs):
            hx[x_off[c]:x_off[c] + x.numel()].copy_(x.reshape(-1).cpu())
        hy = torch.empty(oo, dtype=torch.bfloat16).pin_memory()
        dxf = torch.empty(xo, dtype=torch.bfloat16, device=dev)
        dyf = torch.empty(oo, dtype=torch.bfloat16, device=dev)
        dx = [dxf[x_off[c]:x_off[c] + M * K].view(M, K) for c, (M, N, K, *_r) in enumerate(calls)]
        dy = [dyf[o_off[c]:o_off[c] + M * N].view(M, N) for c, (M, N, K, *_r) in enumerate(calls)]
        h2d = xo * 2
        d2h = oo * 2

        def e2e_step(s):
            with torch.cuda.stream(stream):
                dxf.copy_(hx, non_blocking=True)
                ctr = {}
                for c, (M, N, K, *_r) in enumerate(calls):
                    k = ctr.get((N, K), 0)
                    ctr[(N, K)] = k + 1
                    cp = wcopies[(N, K)]
                    wq, wsc = cp[(s * uses[(N, K)] + k) % len(cp)]
                    q, sc = fb.quant_act_per_token_group(dx[c], q=qs[c], scale=ss[c], stream=stream)
                    fb.gemm_a8w8_blockscale(q, sc, wq, wsc, out=dy[c], workspace=workspace, stream=stream,
                                            static_weights=True, **tkw(N))
                hy.copy_(dyf, non_blocking=True)
        for s in range(3):
            e2e_step(s)
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for s in range(e2e_steps):
            e2e_step(s)
        e1.record(stream)
        barrier()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, dev)
        e2e = {"value": round(e2e_ms * 1000.0 / (n_calls * world), 3), "unit": "µs/call",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "api": "fp8_block_scaled_a8w8_b200.quant_act_per_token_group + gemm_a8w8_blockscale (eager); "
                      "one pinned host->device copy of the step's activations and one device->host copy "
                      "of its outputs"}

    if rank == 0:
        det = per_call_detail(fb, torch, calls, cfgs, wcopies, qs, ss, outs, workspace, stream, pk, tkw=tkw) \
            if detail else None
        tot_bytes = float(sum(a8w8_bytes(M, N, K) for (M, N, K, *_r) in calls))
        tot_ms = gemm_ms_per_call * n_calls
        tot_flops = sum(2.0 * M * N * K for (M, N, K, *_r) in calls)
        fp8_peak = 2.0 * pk["bf16_tflops_sustained"]  # fp8 dense = 2x bf16 (nominal 4.5 / 2.25 PFLOP/s)
        hbm_bound = tot_bytes / (pk["hbm_gbs"] * 1e9) >= tot_flops / (fp8_peak * 1e12)
        if hbm_bound:
            achieved = tot_bytes / (tot_ms * 1e-3) / 1e9
            roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                    "frac": round(achieved / pk["hbm_gbs"], 4),
                    "peak_source": f"{pk['source']} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"}
        else:
            achieved = tot_flops / (tot_ms * 1e-3) / 1e12
            roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(fp8_peak, 1), "unit": "TFLOP/s",
                    "frac": round(achieved / fp8_peak, 4),
                    "peak_source": f"2 x {pk['source']} sustained bf16 cuBLAS (fp8/bf16 nominal ratio 2)"}
        key = "gemv_tma" if all(c == "a8w8_gemv_tma" for c in cfgs) else \
            "gemv_umma" if all(c == "a8w8_gemv_umma" for c in cfgs) else \
            "gemm_fp8" if all(c.startswith(("a8w8_tcw", "a8w8_tc2")) for c in cfgs) else \
            "gemm_tc" if all(c.startswith("a8w8_tc_") for c in cfgs) else None
        roof["traffic"] = measured_traffic(key, tot_bytes / n_calls) if key else None
        roof["traffic_note"] = "DRAM bytes per launch (average call), ncu capture in profiles/ scaled by algorithmic bytes"
        roof["kernel"] = "gemm_a8w8_blockscale: " + ", ".join(sorted(set(cfgs)))
        roof["algorithmic_bytes_per_step"] = int(tot_bytes)
        roof["gemm_us_per_step"] = round(tot_ms * 1000.0, 2)
        # the activation quantiser (a1), timed as the block of quant launches in the same graphs
        q_bytes = float(sum(3 * M * K + 4 * M * (K // 128) for (M, N, K, *_r) in calls))
        q_gbs = q_bytes / (quant_block_ms * 1e-3) / 1e9
        quant_roof = {"kernel": "quant_act_per_token_group", "bound": "hbm", "achieved": round(q_gbs, 1),
                      "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": round(q_gbs / pk["hbm_gbs"], 4),
                      "us_per_step": round(quant_block_ms * 1000.0, 2),
                      "algorithmic_bytes_per_step": int(q_bytes),
                      "note": "bf16 read + e4m3 write + fp32 scales per element; at decode M the launches are latency-bound"}
        cpu_line = None
        if cpu and world == 1:
            def gpu_output(c, rows):
                """The call's output recomputed through the public API on copy 0 of its weight
                (the inputs of the timed calls), rows selected, as float64."""
                M, N, K, *_r = calls[c]
                wq0, ws0 = wcopies[(N, K)][0]
                with torch.cuda.stream(stream):
                    q, sc = fb.quant_act_per_token_group(xs[c], stream=stream)
                    y = fb.gemm_a8w8_blockscale(q, sc, wq0, ws0, workspace=workspace, stream=stream, **tkw(N))
                stream.synchronize()
                return y.float().cpu().numpy().astype(np.float64)[rows]
            cpu_line = cpu_baseline(workload, calls, [x.cpu() for x in xs], gpu_output)
        line = {
            "metric": METRIC, "value": round(step_ms * 1000.0 / (n_calls * world), 3), "unit": "µs/call",
            "n_gpus": world, "steps": steps, "warmup": warmup, "ms_per_step": round(step_ms, 4),
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "e4m3 x e4m3 -> f32 -> bf16",
            "data": "synthetic (seeded N(0,1) activations, N(0,0.02) weights; no dataset)",
            "config": {"workload": workload if not shape else "shape " + shape,
                       "description": inputs.WORKLOADS[workload] if not shape else "one a8w8 call shape M,N,K",
                       "calls_per_step": n_calls,
                       "weight_rotation_mib": ROTATE_BYTES >> 20,
                       "weight_layout": "16 KiB tiles (tile_weight)" if tiled else "[N, K] row-major",
                       "l2": "working set per step >> 126 MB L2 (rotated weights); no flush needed",
                       "parallelism": f"replicas x{world}", "timing": "CUDA graphs replayed, CUDA events, max over ranks"},
            "roofline": roof, "quant_roofline": quant_roof,
            "cpu_baseline": cpu_line, "e2e": e2e, "gpu_launches": 2 * n_calls * steps,
            "clocks": clk, "dispatch": {**census, "table_hash": fb.dispatch_table_hash(),
                                        "padded_m_drift": padded_m_drift(fb.dispatch_dump_json(), fb.OP_A8W8_BLOCKSCALE)},
            "detail": det,
        }
        if cpu_line is not None and "accuracy" in cpu_line:
            line["accuracy"] = cpu_line.pop("accuracy")
        if det:
            hot = [d["hot_us"] for d in det if d.get("hot_us") is not None]
            per_shape = {(d["M"], d["N"], d["K"]): d for d in det}
            cold_mean = float(np.mean([per_shape[(M, N, K)]["us"] for (M, N, K, *_r) in calls]))
            hot_mean = float(np.mean([per_shape[(M, N, K)]["hot_us"] for (M, N, K, *_r) in calls])) if hot else None
            line["hot"] = {"value": round(hot_mean, 3) if hot_mean else None, "unit": "µs/call",
                           "cold_value": round(cold_mean, 3),
                           "protocol": "GEMM only, 20 back-to-back calls per shape in a CUDA graph: hot = one weight "
                                       "copy (L2-resident when it fits), cold = rotated over >= 512 MiB; mean over "
                                       "the workload's calls"}
            one = per_shape.get((1, 5120, 6144))
            if one is not None:
                line["single_call"] = {"workload": "decode_m1_n5120_k6144", "M": 1, "N": 5120, "K": 6144,
                                       "us": one["us"], "hot_us": one.get("hot_us"), "GBps": one["GBps"],
                                       "roofline_frac": one["roofline_frac"], "cfg": one["cfg"]}
    else:
        line = None
    for g in graphs:
        del g
    graphs.clear()
    return line


def per_call_detail(fb, torch, calls, cfgs, wcopies, qs, ss, outs, workspace, stream, pk, R=20, rounds=7,
                    tkw=lambda N: {}):
    """us/call of every distinct call shape: R back-to-back calls in one CUDA graph, median
    over rounds interleaved across shapes ([aiter#7752] "Kernel": graph replay, median of
    interleaved rounds), once on weight copies rotated over >= 512 MiB (cold: every call
    reads its weights from HBM) and once on a single copy (hot), as the pages report both."""
    seen, idx = set(), []
    for c, (M, N, K, *_r) in enumerate(calls):
        if (M, N, K) not in seen:
            seen.add((M, N, K))
            idx.append(c)
    graphs = {}
    with torch.cuda.stream(stream):
        for c in idx:
            M, N, K, *_r = calls[c]
            cp = wcopies[(N, K)]
            for kind in ("cold", "hot"):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    for r in range(R):
                        wq, wsc = cp[r % len(cp)] if kind == "cold" else cp[0]
                        fb.gemm_a8w8_blockscale(qs[c], ss[c], wq, wsc, out=outs[c], workspace=workspace,
                                                stream=stream, static_weights=True, **tkw(N))
                graphs[(c, kind)] = g
    times = {k: [] for k in graphs}
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(rounds):
        for k, g in graphs.items():
            with torch.cuda.stream(stream):
                e0.record(stream)
                g.replay()
                e1.record(stream)
            e1.synchronize()
            times[k].append(e0.elapsed_time(e1) * 1000.0 / R)
    out = []
    for c in idx:
        M, N, K, *_r = calls[c]
        t = sorted(times[(c, "cold")])
        us = t[len(t) // 2]
        th = sorted(times[(c, "hot")])
        by = a8w8_bytes(M, N, K)
        fl = 2.0 * M * N * K
        # timed alone in short bursts: the burst peaks (HBM copy; fp8 = 2 x burst bf16)
        roof_us = max(by / (pk["hbm_gbs"] * 1e3), fl / (2 * pk["bf16_tflops"] * 1e6))
        out.append({"M": M, "N": N, "K": K, "cfg": cfgs[c], "us": round(us, 3),
                    "iqr_us": round(t[(3 * len(t)) // 4] - t[len(t) // 4], 3), "hot_us": round(th[len(th) // 2], 3),
                    "GBps": round(by / us / 1e3, 1), "TFLOPS": round(fl / us / 1e6, 2),
                    "roofline_frac": round(roof_us / us, 3)})
    graphs.clear()
    return out


def padded_m_drift(census, op):
    """Padded-M drift of the census ([cookbook#8] "Two amplifiers": M = 6016 runs the row
    tuned for 8192): lookups whose hit came from a row at a padded M other than the exact
    M, their share of all hits, and the distinct (M, padded_M) pairs."""
    hits = [r for r in census if r["op"] == op and r["hit"]]
    drifted = [r for r in hits if r["padded_M"] != r["M"]]
    n_hits = sum(r["count"] for r in hits)
    n_drift = sum(r["count"] for r in drifted)
    return {"lookups": n_drift, "share_of_hits": round(n_drift / n_hits, 4) if n_hits else 0.0,
            "distinct": len({(r["M"], r["padded_M"]) for r in drifted}),
            "max_ratio": round(max((r["padded_M"] / r["M"] for r in drifted), default=1.0), 3)}


# --------------------------------------------------------------------------- CPU oracle
def _oracle_call(x, N, K, i, wcache):
    """The oracle on one call: activations x (float32 array of bf16 values), the call's
    weight quantised by the oracle (set-up, untimed). Returns (seconds, ref float64)."""
    from oracle import gemm as ogemm, quant as oquant
    key = (N, K)
    if key not in wcache:
        w = inputs.weight_f32(N, K, inputs.decode_seed_w(i)).numpy()
        wcache[key] = oquant.quant_weight_block128(w)  # set-up, untimed
    W_q, w_s = wcache[key]
    t0 = time.perf_counter()
    A_q, a_s = oquant.quant_act_per_token_group(x)
    ref, _ = ogemm.gemm_a8w8_blockscale(A_q, a_s, W_q, w_s)
    return time.perf_counter() - t0, ref


def _threads():
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 1) for d in threadpool_info() if d.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return os.cpu_count() or 1


def _host():
    """CPU model and the cores this process may run on (sched_getaffinity)."""
    model = None
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    try:
        aff = len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        aff = os.cpu_count()
    return {"cpu_model": model, "affinity_cores": aff}


def _accuracy(pairs):
    """rel L2 ([aiter#7752] "Kernel") and error ratio ([aiter#7247] "Test Result"; atol =
    1e-2 x rms of the reference, rtol = 1e-2) of GPU outputs against the oracle, over all
    compared outputs."""
    from oracle import metrics as ometrics
    y = np.concatenate([p[0].ravel() for p in pairs])
    r = np.concatenate([p[1].ravel() for p in pairs])
    rms = float(np.sqrt(np.mean(r * r))) if r.size else 0.0
    return {"rel_l2": round(ometrics.rel_l2(y, r), 6),
            "error_ratio": round(ometrics.error_ratio(y, r, atol=1e-2 * rms, rtol=1e-2), 6),
            "atol": round(1e-2 * rms, 8), "rtol": 1e-2, "outputs": int(y.size),
            "reference": "CPU oracle in float64 (unrounded)"}


def cpu_baseline(workload, calls=None, xs=None, gpu_output=None, budget_s=20.0):
    """The oracle as it stands, timed on the host on a bounded sample of the workload. With
    the timed calls' activations (xs) and a way to recompute a call's GPU output, the same
    oracle results also give the accuracy of the GPU outputs on that sample."""
    if calls is None:
        calls = workload_calls(workload)
    order = list(np.random.default_rng(0).permutation(len(calls)))
    wcache = {}
    spent, done, pairs = 0.0, [], []
    for c in order:
        M, N, K, i, j, o = calls[c]
        m = min(M, 64)  # rows of a large-M call: the oracle is row-separable; time per row is scaled below
        rows = np.arange(m) if m == M else np.unique(np.concatenate([np.arange(m // 2), np.arange(M - m + m // 2, M)]))
        if xs is not None:
            x = xs[c].float().numpy()[rows]
        else:
            x = inputs.activation_bf16(M, K, inputs.decode_seed_a(i, j), outliers=o).float().numpy()[rows]
        dt, ref = _oracle_call(x, N, K, i, wcache)
        if gpu_output is not None:
            pairs.append((gpu_output(c, rows), ref))
        spent += dt
        done.append(dt * M / len(rows))
        if spent > budget_s:
            break
    us = float(np.mean(done)) * 1e6
    out = {"value": round(us, 1), "unit": "µs/call", "cores": _threads(), **_host(), "kind": "oracle",
           "sample": f"{len(done)} of {len(calls)} calls of the {workload} workload (random order), quant + GEMM in "
                     f"float64{'; calls with M > 64 timed on 64 rows (first and last) and scaled by M/64' if any(c[0] > 64 for c in calls) else ''}"}
    if pairs:
        out["accuracy"] = {**_accuracy(pairs), "sample": f"the same {len(pairs)} calls, outputs of the timed inputs"}
    return out


# --------------------------------------------------------------------------- bf16 small-N workload
BF16_METRIC = "bf16 GEMM µs/call, TFLOPS & HBM GB/s (cold weights) vs roofline"


BF16_WORKLOADS = ("bf16_small_n", "lm_head")


def bf16_calls(workload="bf16_small_n"):
    """(M, N, K, out_fp32, nk_index, m_index) of a bf16 workload."""
    if workload == "lm_head":
        N, K = inputs.LM_HEAD_NK
        return [(M, N, K, False, 0, j) for j, M in enumerate(inputs.LM_HEAD_MS)]
    return [(M, N, K, f32, i, j) for i, (N, K, f32) in enumerate(inputs.BF16_NK) for j, M in enumerate(inputs.BF16_MS)]


def _oracle_bf16_call(M, N, K, f32, i, j, wcache):
    from oracle import gemm as ogemm
    if (N, K) not in wcache:
        wcache[(N, K)] = inputs.weight_bf16(N, K, inputs.decode_seed_w(i)).float().numpy()  # set-up, untimed
    a = inputs.activation_bf16(M, K, inputs.decode_seed_a(i, j)).float().numpy()
    t0 = time.perf_counter()
    ogemm.gemm_bf16(a, wcache[(N, K)], out_fp32=f32)
    return time.perf_counter() - t0


def cpu_baseline_bf16(workload="bf16_small_n", budget_s=20.0):
    calls = bf16_calls(workload)
    order = list(np.random.default_rng(0).permutation(len(calls)))
    wcache, spent, done = {}, 0.0, []
    for c in order:
        M, N, K, f32, i, j = calls[c]
        m = min(M, 64)  # the oracle is row-separable: large-M calls are timed on 64 rows and scaled
        dt = _oracle_bf16_call(m, N, K, f32, i, j, wcache)
        spent += dt
        done.append(dt * M / m)
        if spent > budget_s:
            break
    return {"value": round(float(np.mean(done)) * 1e6, 1), "unit": "µs/call", "cores": _threads(), **_host(),
            "kind": "oracle",
            "sample": f"{len(done)} of {len(calls)} calls of the {workload} workload (random order), float64 "
                      "matmul; calls with M > 64 timed on 64 rows and scaled by M/64"}


def measure_bf16(args, world, rank, dev, steps, warmup, detail, e2e_steps, cpu, workload="bf16_small_n"):
    """The JSON line of a bf16 workload (rank 0; None elsewhere)."""
    import torch
    import torch.distributed as dist

    import fp8_block_scaled_a8w8_b200 as fb

    fb.lib()
    pk = peaks()
    calls = bf16_calls(workload)
    n_calls = len(calls)
    uses, maxm = {}, {}
    for (M, N, K, f32, i, j) in calls:
        uses[(N, K)] = uses.get((N, K), 0) + 1
        maxm[(N, K)] = max(maxm.get((N, K), 0), M)
    wcopies, bx, bo = {}, {}, {}
    for (M, N, K, f32, i, j) in calls:
        if (N, K) in wcopies:
            continue
        w = inputs.weight_bf16(N, K, inputs.decode_seed_w(i)).to(dev)
        # one distinct copy per use within a step (each call reads cold weights); between two
        # steps the large-M calls stream > 1 GB of activations, far above the 126 MB L2
        wcopies[(N, K)] = [w] + [w.clone() for _ in range(uses[(N, K)] - 1)]
        bx[(N, K)] = inputs.activation_bf16(maxm[(N, K)], K, inputs.decode_seed_a(i, 0)).to(dev)
        bo[(N, K)] = torch.empty((maxm[(N, K)], N), dtype=torch.float32 if f32 else torch.bfloat16, device=dev)
    xs = [bx[(N, K)][:M] for (M, N, K, *_r) in calls]
    outs = [bo[(N, K)][:M] for (M, N, K, *_r) in calls]
    workspace = torch.zeros(max(256, max(fb.workspace_bytes(fb.OP_BF16, M, N, K) for (M, N, K, *_r) in calls)),
                            dtype=torch.uint8, device=dev)
    cfgs = [fb.dispatch_lookup(fb.OP_BF16, M, N, K)[1] for (M, N, K, *_r) in calls]
    period = 1
    stream = torch.cuda.Stream(device=dev)

    def step_launches(s, ev=None):
        if ev is not None:
            ev[0].record(stream)
        ctr = {}
        for c, (M, N, K, f32, *_r) in enumerate(calls):
            k = ctr.get((N, K), 0)
            ctr[(N, K)] = k + 1
            cp = wcopies[(N, K)]
            fb.gemm_bf16(xs[c], cp[(s * uses[(N, K)] + k) % len(cp)], out_fp32=f32, out=outs[c], workspace=workspace,
                         stream=stream)
        if ev is not None:
            ev[1].record(stream)

    events = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)] for _ in range(period)]
    graphs = []
    fb.dispatch_reset_stats()
    with torch.cuda.stream(stream):
        for ph in range(period):
            step_launches(ph)
        stream.synchronize()
        for ph in range(period):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                step_launches(ph, events[ph])
            graphs.append(g)
    torch.cuda.synchronize()
    census = fb.dispatch_stats(fb.OP_BF16)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    with torch.cuda.stream(stream):
        for s in range(warmup):
            graphs[s % period].replay()
    barrier()
    clocks = ClockSampler(dev.index)
    if rank == 0:
        clocks.start()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    t_start.record(stream)
    for s in range(steps):
        with torch.cuda.stream(stream):
            graphs[(warmup + s) % period].replay()
    t_end.record(stream)
    barrier()
    clk = clocks.stop() if rank == 0 else None
    step_ms = max_over_ranks(t_start.elapsed_time(t_end) / steps, dev)

    e2e = None
    if e2e_steps > 0:
        e2e_steps = min(e2e_steps, 5)
        hx = [x.cpu().pin_memory() for x in xs]
        hy = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs]
        dxb = {k: torch.empty_like(v) for k, v in bx.items()}
        dx = [dxb[(N, K)][:M] for (M, N, K, *_r) in calls]
        h2d = sum(x.numel() * x.element_size() for x in xs)
        d2h = sum(o.numel() * o.element_size() for o in outs)

        def e2e_step(s):
            with torch.cuda.stream(stream):
                ctr = {}
                for c, (M, N, K, f32, *_r) in enumerate(calls):
                    dx[c].copy_(hx[c], non_blocking=True)
                    k = ctr.get((N, K), 0)
                    ctr[(N, K)] = k + 1
                    cp = wcopies[(N, K)]
                    fb.gemm_bf16(dx[c], cp[(s * uses[(N, K)] + k) % len(cp)], out_fp32=f32, out=outs[c],
                                 workspace=workspace, stream=stream)
                    hy[c].copy_(outs[c], non_blocking=True)
        for s in range(2):
            e2e_step(s)
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for s in range(e2e_steps):
            e2e_step(s)
        e1.record(stream)
        barrier()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, dev)
        e2e = {"value": round(e2e_ms * 1000.0 / (n_calls * world), 3), "unit": "µs/call",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "api": "fp8_block_scaled_a8w8_b200.gemm_bf16 (eager)"}

    if rank == 0:
        gemm_ms = float(np.mean([events[ph][0].elapsed_time(events[ph][1]) for ph in sorted(
            {(warmup + s) % period for s in range(steps)})]))
        tot_bytes = float(sum(bf16_bytes(M, N, K, f32) for (M, N, K, f32, *_r) in calls))
        tot_flops = float(sum(2.0 * M * N * K for (M, N, K, *_r) in calls))
        peak_tf = pk["bf16_tflops_sustained"]
        t_hbm = tot_bytes / (pk["hbm_gbs"] * 1e9)
        t_tc = tot_flops / (peak_tf * 1e12)
        t_roof = sum(max(bf16_bytes(M, N, K, f32) / (pk["hbm_gbs"] * 1e9), 2.0 * M * N * K / (peak_tf * 1e12))
                     for (M, N, K, f32, *_r) in calls)
        if t_hbm >= t_tc:
            ach = tot_bytes / (gemm_ms * 1e-3) / 1e9
            roof = {"bound": "hbm", "achieved": round(ach, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                    "frac": round(ach / pk["hbm_gbs"], 4),
                    "peak_source": f"{pk['source']} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"}
        else:
            ach = tot_flops / (gemm_ms * 1e-3) / 1e12
            roof = {"bound": "tensor", "achieved": round(ach, 1), "peak": peak_tf, "unit": "TFLOP/s",
                    "frac": round(ach / peak_tf, 4),
                    "peak_source": f"{pk['source']} sustained bf16 cuBLAS (MEASURED_PEAKS.json bf16_tflops_sustained)"}
        roof["traffic"] = None
        roof["roofline_time_frac"] = round(t_roof / (gemm_ms * 1e-3), 4)
        roof["kernel"] = "gemm_bf16: " + ", ".join(sorted(set(cfgs)))
        roof["gemm_us_per_step"] = round(gemm_ms * 1000.0, 2)
        det = None
        if detail:
            det = []
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            for c, (M, N, K, f32, *_r) in enumerate(calls):
                cp = wcopies[(N, K)]
                g = torch.cuda.CUDAGraph()
                with torch.cuda.stream(stream):
                    with torch.cuda.graph(g, stream=stream):
                        for r in range(20):
                            fb.gemm_bf16(xs[c], cp[r % len(cp)], out_fp32=f32, out=outs[c], workspace=workspace,
                                         stream=stream)
                    ts = []
                    for _ in range(5):
                        e0.record(stream)
                        g.replay()
                        e1.record(stream)
                        e1.synchronize()
                        ts.append(e0.elapsed_time(e1) * 1000.0 / 20)
                del g
                us = sorted(ts)[len(ts) // 2]
                by, fl = bf16_bytes(M, N, K, f32), 2.0 * M * N * K
                roof_us = max(by / (pk["hbm_gbs"] * 1e3), fl / (peak_tf * 1e6))
                det.append({"M": M, "N": N, "K": K, "out": "f32" if f32 else "bf16", "cfg": cfgs[c],
                               "us": round(us, 3), "GBps": round(by / us / 1e3, 1), "TFLOPS": round(fl / us / 1e6, 2),
                               "roofline_frac": round(roof_us / us, 3)})
        cpu_line = cpu_baseline_bf16(workload) if (cpu and world == 1) else None
        line = {
            "metric": BF16_METRIC, "value": round(step_ms * 1000.0 / (n_calls * world), 3), "unit": "µs/call",
            "n_gpus": world, "steps": steps, "warmup": warmup, "ms_per_step": round(step_ms, 4),
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16 x bf16 -> f32",
            "data": "synthetic (seeded N(0,1) activations, N(0,0.02) weights; no dataset)",
            "config": {"workload": workload, "description": inputs.WORKLOADS[workload],
                       "calls_per_step": n_calls, "weight_rotation_mib": ROTATE_BYTES >> 20,
                       "l2": "one weight copy per use within a step; > 1 GB of activations streamed per step (L2 126 MB)",
                       "parallelism": f"replicas x{world}", "timing": "CUDA graphs replayed, CUDA events, max over ranks"},
            "roofline": roof, "cpu_baseline": cpu_line, "e2e": e2e, "gpu_launches": n_calls * steps,
            "clocks": clk, "dispatch": {**census, "table_hash": fb.dispatch_table_hash()}, "detail": det,
        }
    else:
        line = None
    for g in graphs:
        del g
    graphs.clear()
    return line


# --------------------------------------------------------------------------- MX32 workloads
MX_METRIC = "MX32 a8w8 GEMM µs/call, TFLOPS & HBM GB/s (cold weights) vs roofline"


def mx_calls(workload):
    """(batch, M, N, K) of an MX32 workload."""
    if workload == "mx32_batched":
        b, N, K = inputs.MX32_BATCHED
        return [(b, M, N, K) for M in inputs.MX32_BATCHED_MS]
    return [(1, M, N, K) for (N, K) in inputs.MX32_NK for M in inputs.MX32_MS]


def mx_bytes(b, M, N, K):
    """A + a_e8m0 + W + w_e8m0 + out."""
    return b * (M * K + M * (K // 32) + N * K + ((N + 31) // 32) * (K // 32) + 2 * M * N)


def measure_mx(args, world, rank, dev, workload, steps, warmup, detail):
    """An MX32 workload: calls on weights rotated over >= 512 MiB of copies, one CUDA graph
    per rotation phase (rank 0's line; None elsewhere)."""
    import torch

    import fp8_block_scaled_a8w8_b200 as fb

    fb.lib()
    pk = peaks()
    calls = mx_calls(workload)
    shapes = sorted({(b, N, K) for (b, M, N, K) in calls})
    wcopies, acts = {}, {}
    for si, (b, N, K) in enumerate(shapes):
        uses = sum(1 for c in calls if (c[0], c[2], c[3]) == (b, N, K))
        w = inputs.weight_f32(b * N, K, 700 + si).to(dev)
        wq, we = fb.quant_weight_mx32(w)
        del w
        # per batch the 32-row blocks must not straddle batches: N % 32 == 0 for these shapes
        wq, we = wq.view(b, N, K), we.view(b, (N + 31) // 32, K // 32)
        per = wq.numel() + we.numel()
        n = max(1, math.ceil(ROTATE_BYTES / per))
        n = uses * math.ceil(n / uses)
        wcopies[(b, N, K)] = [(wq, we)] + [(wq.clone(), we.clone()) for _ in range(n - 1)]
    for (b, M, N, K) in calls:
        if (b, M, K) not in acts:
            x = inputs.activation_bf16(b * M, K, 800 + M + K).to(dev)
            q, e = fb.quant_act_mx32(x)
            acts[(b, M, K)] = (q.view(b, M, K) if b > 1 else q, e.view(b, M, K // 32) if b > 1 else e)
    outs = [torch.empty(((b,) if b > 1 else ()) + (M, N), dtype=torch.bfloat16, device=dev) for (b, M, N, K) in calls]
    ws = torch.zeros(max(256, max(fb.mx32_workspace_bytes(b, M, N, K) for (b, M, N, K) in calls)), dtype=torch.uint8,
                     device=dev)
    period = 1
    for key, cp in wcopies.items():
        u = sum(1 for c in calls if (c[0], c[2], c[3]) == key)
        period = period * (len(cp) // u) // math.gcd(period, len(cp) // u)
    stream = torch.cuda.Stream(device=dev)

    def weights(s, c):
        b, M, N, K = calls[c]
        k = sum(1 for j in range(c) if (calls[j][0], calls[j][2], calls[j][3]) == (b, N, K))
        u = sum(1 for j in range(len(calls)) if (calls[j][0], calls[j][2], calls[j][3]) == (b, N, K))
        cp = wcopies[(b, N, K)]
        wq, we = cp[(s * u + k) % len(cp)]
        return (wq[0], we[0]) if b == 1 else (wq, we)

    def step(s, ev=None):
        if ev is not None:
            ev[0].record(stream)
        for c, (b, M, N, K) in enumerate(calls):
            q, e = acts[(b, M, K)]
            wq, we = weights(s, c)
            fb.gemm_a8w8_mx32(q, e, wq, we, out=outs[c], workspace=ws, stream=stream)
        if ev is not None:
            ev[1].record(stream)

    events = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)] for _ in range(period)]
    graphs = []
    with torch.cuda.stream(stream):
        for ph in range(period):
            step(ph)
        stream.synchronize()
        for ph in range(period):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                step(ph, events[ph])
            graphs.append(g)
        for s_ in range(warmup):
            graphs[s_ % period].replay()
    torch.cuda.synchronize()
    clocks = ClockSampler(dev.index)
    if rank == 0:
        clocks.start()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t0.record(stream)
    for s_ in range(steps):
        with torch.cuda.stream(stream):
            graphs[(warmup + s_) % period].replay()
    t1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop() if rank == 0 else None
    step_ms = max_over_ranks(t0.elapsed_time(t1) / steps, dev)
    line = None
    if rank == 0:
        gemm_ms = float(np.mean([events[ph][0].elapsed_time(events[ph][1]) for ph in sorted(
            {(warmup + s_) % period for s_ in range(steps)})]))
        tot_bytes = float(sum(mx_bytes(*c) for c in calls))
        tot_flops = float(sum(2.0 * b * M * N * K for (b, M, N, K) in calls))
        fp8_peak = 2.0 * pk["bf16_tflops_sustained"]
        t_roof = sum(max(mx_bytes(*c) / (pk["hbm_gbs"] * 1e9), 2.0 * c[0] * c[1] * c[2] * c[3] / (fp8_peak * 1e12))
                     for c in calls)
        if tot_bytes / (pk["hbm_gbs"] * 1e9) >= tot_flops / (fp8_peak * 1e12):
            ach = tot_bytes / (gemm_ms * 1e-3) / 1e9
            roof = {"bound": "hbm", "achieved": round(ach, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                    "frac": round(ach / pk["hbm_gbs"], 4)}
        else:
            ach = tot_flops / (gemm_ms * 1e-3) / 1e12
            roof = {"bound": "tensor", "achieved": round(ach, 1), "peak": round(fp8_peak, 1), "unit": "TFLOP/s",
                    "frac": round(ach / fp8_peak, 4),
                    "peak_source": "2 x measured sustained bf16 cuBLAS (fp8/bf16 nominal ratio 2)"}
        roof.update({"roofline_time_frac": round(t_roof / (gemm_ms * 1e-3), 4), "traffic": None,
                     "kernel": "gemm_mx_kernel (tcgen05.mma kind::mxf8f6f4.block_scale)",
                     "gemm_us_per_step": round(gemm_ms * 1000.0, 2)})
        det = None
        if detail:
            det = []
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            for c, (b, M, N, K) in enumerate(calls):
                q, e = acts[(b, M, K)]
                cp = wcopies[(b, N, K)]
                g = torch.cuda.CUDAGraph()
                with torch.cuda.stream(stream):
                    with torch.cuda.graph(g, stream=stream):
                        for r in range(20):
                            wq, we = cp[r % len(cp)]
                            if b == 1:
                                wq, we = wq[0], we[0]
                            fb.gemm_a8w8_mx32(q, e, wq, we, out=outs[c], workspace=ws, stream=stream)
                    ts = []
                    for _ in range(5):
                        e0.record(stream)
                        g.replay()
                        e1.record(stream)
                        e1.synchronize()
                        ts.append(e0.elapsed_time(e1) * 1000.0 / 20)
                del g
                us = sorted(ts)[len(ts) // 2]
                by, fl = mx_bytes(b, M, N, K), 2.0 * b * M * N * K
                roof_us = max(by / (pk["hbm_gbs"] * 1e3), fl / (2 * pk["bf16_tflops"] * 1e6))
                det.append({"batch": b, "M": M, "N": N, "K": K, "us": round(us, 3), "GBps": round(by / us / 1e3, 1),
                            "TFLOPS": round(fl / us / 1e6, 2), "roofline_frac": round(roof_us / us, 3)})
        line = {"metric": MX_METRIC, "value": round(step_ms * 1000.0 / (len(calls) * world), 3), "unit": "µs/call",
                "ms_per_step": round(step_ms, 4), "steps": steps, "warmup": warmup, "dtype": "e4m3 x e4m3 (E8M0) -> f32",
                "config": {"workload": workload, "description": inputs.WORKLOADS[workload], "calls_per_step": len(calls),
                           "weight_rotation_mib": ROTATE_BYTES >> 20},
                "roofline": roof, "gpu_launches": len(calls) * steps, "clocks": clk, "detail": det}
    graphs.clear()
    return line


# --------------------------------------------------------------------------- fused norm + quant workload
NORM_METRIC = "add_rmsnorm_quant µs/call & HBM GB/s vs roofline"


def norm_bytes(M, K):
    """x + residual read, residual_out written (bf16), codes written, scales written, gamma read."""
    return 7 * M * K + 4 * M * (K // 128) + 2 * K


def measure_norm(args, world, rank, dev, steps, warmup):
    """The fused residual add + RMSNorm + activation quantisation over the decode and prefill
    token counts (rank 0's line; None elsewhere)."""
    import torch

    import fp8_block_scaled_a8w8_b200 as fb

    fb.lib()
    pk = peaks()
    calls = [(M, K) for K in inputs.NORM_KS for M in inputs.NORM_MS]
    bufs = []
    for i, (M, K) in enumerate(calls):
        x = inputs.activation_bf16(M, K, 300 + i).to(dev)
        r = inputs.activation_bf16(M, K, 400 + i).to(dev)
        g = (1.0 + 0.1 * inputs.activation_bf16(1, K, 500 + i).float()).to(torch.bfloat16)[0].to(dev)
        bufs.append((x, r, g, torch.empty_like(x), torch.empty((M, K), dtype=torch.float8_e4m3fn, device=dev),
                     torch.empty((M, K // 128), dtype=torch.float32, device=dev)))
    stream = torch.cuda.Stream(device=dev)
    ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]

    def step(e=None):
        if e is not None:
            e[0].record(stream)
        for (x, r, g, ro, q, s) in bufs:
            fb.add_rmsnorm_quant(x, r, g, 1e-6, residual_out=ro, q=q, scale=s, stream=stream)
        if e is not None:
            e[1].record(stream)

    with torch.cuda.stream(stream):
        step()
        stream.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            step(ev)
        for _ in range(warmup):
            graph.replay()
    torch.cuda.synchronize()
    clocks = ClockSampler(dev.index)
    if rank == 0:
        clocks.start()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t0.record(stream)
    for _ in range(steps):
        with torch.cuda.stream(stream):
            graph.replay()
    t1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop() if rank == 0 else None
    step_ms = max_over_ranks(t0.elapsed_time(t1) / steps, dev)
    line = None
    if rank == 0:
        tot = float(sum(norm_bytes(M, K) for M, K in calls))
        ms = ev[0].elapsed_time(ev[1])
        ach = tot / (ms * 1e-3) / 1e9
        detail = []
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for (M, K), (x, r, g, ro, q, s) in zip(calls, bufs):
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.stream(stream):
                with torch.cuda.graph(gr, stream=stream):
                    for _ in range(20):
                        fb.add_rmsnorm_quant(x, r, g, 1e-6, residual_out=ro, q=q, scale=s, stream=stream)
                ts = []
                for _ in range(5):
                    e0.record(stream)
                    gr.replay()
                    e1.record(stream)
                    e1.synchronize()
                    ts.append(e0.elapsed_time(e1) * 1000.0 / 20)
            del gr
            us = sorted(ts)[len(ts) // 2]
            detail.append({"M": M, "K": K, "us": round(us, 3), "GBps": round(norm_bytes(M, K) / us / 1e3, 1),
                           "roofline_frac": round(norm_bytes(M, K) / (pk["hbm_gbs"] * 1e3) / us, 3),
                           "note": "20 back-to-back calls on the same buffers (hot in L2 when they fit)"})
        line = {"metric": NORM_METRIC, "value": round(step_ms * 1000.0 / (len(calls) * world), 3), "unit": "µs/call",
                "ms_per_step": round(step_ms, 4), "steps": steps, "warmup": warmup, "dtype": "bf16 -> f32 -> e4m3",
                "config": {"workload": "add_rmsnorm_quant", "description": inputs.WORKLOADS["add_rmsnorm_quant"],
                           "calls_per_step": len(calls),
                           "l2": f"{tot / 1e6:.0f} MB moved per step (> 126 MB L2)"},
                "roofline": {"bound": "hbm", "achieved": round(ach, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                             "frac": round(ach / pk["hbm_gbs"], 4), "traffic": None,
                             "kernel": "add_rmsnorm_quant_kernel", "algorithmic_bytes_per_step": int(tot)},
                "gpu_launches": len(calls) * steps, "clocks": clk, "detail": detail}
    del graph
    return line


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if world > 1 and rank != 0:
        return
    if args.workload in BF16_WORKLOADS:
        return run_reference_bf16(args, world)
    if args.workload == "add_rmsnorm_quant":
        return run_reference_norm(args, world)
    if args.workload in ("mx32", "mx32_batched"):
        return run_reference_mx(args, world)
    calls = workload_calls(args.workload)
    wcache = {}

    def one(c):
        M, N, K, i, j, o = calls[c % len(calls)]
        m = min(M, 64)  # row-separable: large-M calls timed on 64 rows and scaled by M/64
        x = inputs.activation_bf16(m, K, inputs.decode_seed_a(i, j), outliers=o).float().numpy()
        return _oracle_call(x, N, K, i, wcache)[0] * M / m

    for s in range(args.warmup):
        one(s)
    times = [one(args.warmup + s) for s in range(args.steps)]
    us = float(np.mean(times)) * 1e6
    cores = _threads()
    line = {"impl": "reference", "metric": METRIC, "value": round(us, 1), "unit": "µs/call", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(us / 1000.0, 3), "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "description": inputs.WORKLOADS[args.workload]},
            "cpu_baseline": {"value": round(us, 1), "unit": "µs/call", "cores": cores, **_host(), "kind": "oracle",
                             "sample": f"one call per step, cycling through the {args.workload} calls; M > 64 timed "
                                       "on 64 rows and scaled"},
            "e2e": {"value": round(us, 1), "unit": "µs/call", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_reference_norm(args, world):
    """The oracle's fused residual add + RMSNorm + quantisation, one call per step (M > 64
    timed on 64 rows and scaled by M / 64: the step is row-separable)."""
    from oracle import norm as onorm
    calls = [(M, K) for K in inputs.NORM_KS for M in inputs.NORM_MS]

    def one(c):
        M, K = calls[c % len(calls)]
        m = min(M, 64)
        x = inputs.activation_bf16(m, K, 300 + c % len(calls)).float().numpy()
        r = inputs.activation_bf16(m, K, 400 + c % len(calls)).float().numpy()
        g = np.ones(K)
        t0 = time.perf_counter()
        onorm.add_rmsnorm_quant(x, r, g, 1e-6)
        return (time.perf_counter() - t0) * M / m

    for s in range(args.warmup):
        one(s)
    us = float(np.mean([one(args.warmup + s) for s in range(args.steps)])) * 1e6
    line = {"impl": "reference", "metric": NORM_METRIC, "value": round(us, 1), "unit": "µs/call", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(us / 1000.0, 3), "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "add_rmsnorm_quant", "description": inputs.WORKLOADS["add_rmsnorm_quant"]},
            "cpu_baseline": {"value": round(us, 1), "unit": "µs/call", "cores": _threads(), **_host(), "kind": "oracle",
                             "sample": "one call per step, cycling through the calls; M > 64 timed on 64 rows and "
                                       "scaled"},
            "e2e": {"value": round(us, 1), "unit": "µs/call", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_reference_mx(args, world):
    """The oracle's MX32 quantisation + GEMM, one call per step (M > 64 timed on 64 rows and
    scaled by M / 64; the batched form timed on one batch and scaled by b)."""
    from oracle import mx as omx
    calls = mx_calls(args.workload)
    wcache = {}

    def one(c):
        b, M, N, K = calls[c % len(calls)]
        if (N, K) not in wcache:
            wcache[(N, K)] = omx.quant_weight_mx32(inputs.weight_f32(N, K, 700).numpy())  # set-up, untimed
        m = min(M, 64)
        x = inputs.activation_bf16(m, K, 800 + M + K).float().numpy()
        t0 = time.perf_counter()
        Aq, Ae = omx.quant_act_mx32(x)
        omx.gemm_a8w8_mx32(Aq, Ae, *wcache[(N, K)])
        return (time.perf_counter() - t0) * b * M / m

    for s in range(args.warmup):
        one(s)
    us = float(np.mean([one(args.warmup + s) for s in range(args.steps)])) * 1e6
    line = {"impl": "reference", "metric": MX_METRIC, "value": round(us, 1), "unit": "µs/call", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(us / 1000.0, 3), "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "description": inputs.WORKLOADS[args.workload]},
            "cpu_baseline": {"value": round(us, 1), "unit": "µs/call", "cores": _threads(), **_host(), "kind": "oracle",
                             "sample": "one call per step, cycling through the calls; M > 64 timed on 64 rows and "
                                       "scaled, batches scaled by b"},
            "e2e": {"value": round(us, 1), "unit": "µs/call", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_reference_bf16(args, world):
    calls = bf16_calls(args.workload)
    wcache = {}
    for s in range(args.warmup):
        M, N, K, f32, i, j = calls[s % len(calls)]
        _oracle_bf16_call(min(M, 64), N, K, f32, i, j, wcache)
    times = []
    for s in range(args.steps):
        M, N, K, f32, i, j = calls[(args.warmup + s) % len(calls)]
        m = min(M, 64)
        times.append(_oracle_bf16_call(m, N, K, f32, i, j, wcache) * M / m)
    us = float(np.mean(times)) * 1e6
    line = {"impl": "reference", "metric": BF16_METRIC, "value": round(us, 1), "unit": "µs/call", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(us / 1000.0, 3), "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "description": inputs.WORKLOADS[args.workload]},
            "cpu_baseline": {"value": round(us, 1), "unit": "µs/call", "cores": _threads(), **_host(), "kind": "oracle",
                             "sample": f"one call per step, cycling through the {args.workload} calls; M > 64 timed on "
                                       "64 rows and scaled"},
            "e2e": {"value": round(us, 1), "unit": "µs/call", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


SUB_WORKLOADS = {"prefill": 5, "ladder": 3}  # steps of the extra a8w8 workloads of the default run
BF16_SUB_STEPS = 10


def compact(line):
    """The fields of a workload's line that the default run carries for it."""
    keep = ("metric", "value", "unit", "ms_per_step", "steps", "warmup", "dtype", "config", "roofline", "quant_roofline",
            "gpu_launches", "clocks", "dispatch", "detail", "hot")
    return {k: line[k] for k in keep if k in line and line[k] is not None}


def run_gpu(args):
    import torch
    import torch.distributed as dist

    world, rank, dev = init_gpu()
    try:
        if args.workload in BF16_WORKLOADS and not args.shape:
            line = measure_bf16(args, world, rank, dev, args.steps, args.warmup, args.detail, args.e2e_steps,
                                args.cpu_baseline, args.workload)
        elif args.workload == "add_rmsnorm_quant":
            line = measure_norm(args, world, rank, dev, args.steps, args.warmup)
        elif args.workload in ("mx32", "mx32_batched"):
            line = measure_mx(args, world, rank, dev, args.workload, args.steps, args.warmup, args.detail)
        else:
            line = measure_a8w8(args, world, rank, dev, args.workload, args.shape, args.steps, args.warmup,
                                args.detail, args.e2e_steps, args.cpu_baseline)
        torch.cuda.empty_cache()
        if args.all_workloads and args.workload == "decode_sweep" and not args.shape:
            # every other configuration in the same run, each as its own entry with its own
            # roofline (bounded steps; no e2e or CPU legs)
            subs = {}
            for w, k in SUB_WORKLOADS.items():
                subs[w] = measure_a8w8(args, world, rank, dev, w, None, min(args.steps, k), 3, w == "prefill", 0,
                                       False)
                torch.cuda.empty_cache()
            for w in BF16_WORKLOADS:
                subs[w] = measure_bf16(args, world, rank, dev, min(args.steps, BF16_SUB_STEPS), 3, w == "lm_head", 0,
                                       False, w)
                torch.cuda.empty_cache()
            subs["add_rmsnorm_quant"] = measure_norm(args, world, rank, dev, min(args.steps, 20), 3)
            torch.cuda.empty_cache()
            for w in ("mx32", "mx32_batched"):
                subs[w] = measure_mx(args, world, rank, dev, w, min(args.steps, 10), 3, True)
                torch.cuda.empty_cache()
            if rank == 0:
                line["workloads"] = {w: compact(v) for w, v in subs.items()}
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="decode_sweep", choices=list(inputs.WORKLOADS))
    ap.add_argument("--impl", default="fp8bs", choices=["fp8bs", "reference"])
    ap.add_argument("--shape", default=None, help="M,N,K: time one a8w8 call shape instead of a workload")
    ap.add_argument("--layout", choices=["tiled", "standard"], default="tiled",
                    help="a8w8 weight storage: 16 KiB tiles (tile_weight, the default) or [N, K] row-major")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--no-detail", dest="detail", action="store_false",
                    help="skip the per-shape back-to-back timing table (for profiler runs)")
    ap.add_argument("--config", default=None,
                    help="run every a8w8 call of the workload with this kernel configuration (a dispatch row "
                         "per call shape; names from fp8bs_dispatch_list_configs)")
    ap.add_argument("--only", dest="all_workloads", action="store_false",
                    help="decode sweep only: skip the prefill, ladder and bf16 entries of the default run")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
