#!/usr/bin/env python3
"""Benchmark: effective weight GB/s of the small-M quantized matmul on B200.

Metric (MLX issue #4720, "To Reproduce"): weight bytes per call = N*K*bits/8 + N*(K/g)*4
(packed codes + one fp16 scale and bias per group), divided by the time per call, with the
weight copies rotated so that they do not sit in L2.

Headline workload: the 151936-wide LM head (K = 4096, 4-bit, group 64, bf16 x and W ~
N(0, 0.02^2)) at M in {1, 4, 6, 16}, the largest configuration.  Its single 350 MB matrix
is larger than the 126 MB L2, so every call streams its weights from HBM.  One step = one
call per M (4 calls); weights and x are resident in HBM before the timed region; the step
is captured once in a CUDA graph and replayed.

`breakdown` covers the metric as stated, per shape and per M: every M = 1..64 on the three
4-bit shapes (q/o 4096 -> 4096, down 14336 -> 4096, LM head 4096 -> 151936) and M in
{4, 16, 64} on the mixed-precision gate/up and k/v shapes, each cell one CUDA graph of one
call per rotated weight set (>= 2x L2 in total), timed with CUDA events.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line on rank 0.  With --gpus N > 1 (under torchrun), each rank runs the same
per-GPU work on its own GPU (independent problems, no collective on the data path: weak
scaling); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "effective weight GB/s (and % of HBM roofline) per shape vs M=1..64, 1\u00d7B200"
WORKLOAD = "lmhead"
BENCH_MS = (1, 4, 6, 16)
GATED = ("qo", "down", "lmhead")          # every M = 1..64
MIXED = ("gateup_6b", "gateup_8b", "kv_6b", "kv_8b")
MIXED_MS = (4, 16, 64)
NOMINAL_HBM_GBS = 8000.0
KERNEL_NAMES = {1: "qmm_mma_kernel", 2: "qmm_tc_kernel", 3: "qmm_stream_kernel", 4: "qmm_sk_kernel"}
FALLBACK_HBM_GBS = 6650.0
CLOCK_SOAK_S = 2.5  # the step replayed (untimed) while the clocks are sampled, right before timing


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--no-breakdown", action="store_true", help="skip the per-shape, per-M table")
    ap.add_argument("--breakdown-out", default="", help="also write the whole JSON line, indented, here")
    ap.add_argument("--sweep", default="", help="write a per-configuration, per-M GB/s sweep to this "
                    "JSON file instead of running the headline benchmark")
    ap.add_argument("--sweep-configs", default="qo,down,gateup_6b,gateup_8b,kv_6b,kv_8b,lmhead")
    ap.add_argument("--sweep-ms", default="1-64", help="e.g. 1-64 or 1,4,16")
    ap.add_argument("--sweep-plan", default="", help="kernel:split:warps[:flags] override, e.g. 4:1:0:3")
    return ap.parse_args()


# ---------------------------------------------------------------------------- distributed
def init_dist(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    """The largest of the ranks' values (every rank gets it); identity on one process."""
    if world == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_gbs(bytes_per_rank_step: float, ms_per_step: float, world: int) -> float:
    """Whole-job rate for weak scaling: every rank streams the same bytes per step, and the
    step time is the slowest rank's."""
    return bytes_per_rank_step * world / (ms_per_step * 1e-3) / 1e9


# ---------------------------------------------------------------------------- helpers
def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


FALLBACK_TENSOR_TFLOPS = 1400.0  # dense bf16/fp16, sustained under the power cap (earlier measurement)


def tensor_peak():
    """Sustained dense fp16/bf16 tensor rate (TFLOP/s): the measured one, else the fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d.get("bf16_tflops_sustained") or d["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_TENSOR_TFLOPS, "fallback"


def roofline_gbs(wl, M: int, hbm_gbs: float, tflops: float) -> float:
    """The cell's roofline in weight GB/s: the HBM rate, or the tensor rate over the call's
    intensity (2*M*N*K flops per weight byte) where that is lower (4-bit, M >= ~60)."""
    flops_per_byte = 2.0 * M * wl.N * wl.K / wl.weight_bytes()
    return min(hbm_gbs, tflops * 1e3 / flops_per_byte)


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


class ClockSampler:
    """nvidia-smi sampled every 200 ms while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int, enabled: bool):
        self.proc = None
        self.path = os.path.join("/tmp", f"qmm_clocks_{os.getpid()}.csv")
        try:  # the UUID names the physical GPU whatever CUDA_VISIBLE_DEVICES says
            gpu_id = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
        except Exception:
            gpu_id = str(device_index)
        if enabled:
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", f"--id={gpu_id}", f"--query-gpu={self.FIELDS}",
                     "--format=csv,noheader,nounits", "-lms", "200"],
                    stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            except Exception:
                self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append({"sm": float(parts[1]), "max": float(parts[2]), "power": float(parts[3]),
                             "hw": parts[5], "hwt": parts[6], "swt": parts[7], "pcap": parts[8]})
            except ValueError:
                continue
        if not rows:
            return None
        reasons = set()
        for r in rows:
            if r["hw"].lower() == "active":
                reasons.add("hw_slowdown")
            if r["hwt"].lower() == "active":
                reasons.add("hw_thermal_slowdown")
            if r["swt"].lower() == "active":
                reasons.add("sw_thermal_slowdown")
            if r["pcap"].lower() == "active":
                reasons.add("sw_power_cap")
        return {"sm_mhz": statistics.median(r["sm"] for r in rows), "sm_max_mhz": max(r["max"] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows),
                "power_w_max": max(r["power"] for r in rows)}


# ---------------------------------------------------------------------------- our arm
def launches_per_call(q, wl, M: int, plan) -> int:
    """Kernels one call launches, from the library (C ABI qmm_plan_launches): the main kernel
    and the small x kernel where x is prepared in the workspace."""
    return q.plan_launches(M, wl.N, wl.K, wl.bits, wl.group, wl.dtype, plan)


def make_weights(q, wl, dev):
    from bit_quantized_gemm_qmm_b200.inputs import w_input
    weights = []
    for i in range(wl.sets):
        w = w_input(wl.N, wl.K, wl.dtype, i, wl.w_sigma).to(dev)
        weights.append(q.quantize(w, wl.bits, wl.group))
        del w
    return weights


def default_plan(q, wl, M):
    p = q.plan_default(M, wl.N, wl.K, wl.bits, wl.group, wl.dtype)
    p.flags |= q.PLAN_STATIC_WEIGHTS  # weights are written once, before any timed call
    return p


def setup_workload(dev):
    import bit_quantized_gemm_qmm_b200 as q
    from bit_quantized_gemm_qmm_b200.inputs import WORKLOADS, x_input
    wl = WORKLOADS[WORKLOAD]
    weights = make_weights(q, wl, dev)
    xs = {M: x_input(M, wl.K, wl.dtype).to(dev) for M in BENCH_MS}
    ys = {M: torch.empty((M, wl.N), dtype=wl.dtype, device=dev) for M in BENCH_MS}
    plans = {M: default_plan(q, wl, M) for M in BENCH_MS}
    torch.cuda.synchronize()
    return wl, weights, xs, ys, plans


def time_cell(q, wl, weights, M, dev, plan, target_s=0.12):
    """Seconds per call of one (shape, M) cell: a CUDA graph of one call per rotated weight set,
    replayed; the best of three timed batches of replays."""
    from bit_quantized_gemm_qmm_b200.inputs import x_input
    x = x_input(M, wl.K, wl.dtype).to(dev)
    y = torch.empty((M, wl.N), dtype=wl.dtype, device=dev)
    for (P, S, B) in weights:
        q.qmm(x, P, S, B, wl.bits, wl.group, out=y, plan=plan)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for (P, S, B) in weights:
            q.qmm(x, P, S, B, wl.bits, wl.group, out=y, plan=plan)
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g.replay()
    torch.cuda.synchronize()
    e0.record(stream)
    g.replay()
    e1.record(stream)
    e1.synchronize()
    one = max(e0.elapsed_time(e1) * 1e-3, 1e-6)
    reps = max(2, min(200, int(target_s / 3 / one)))
    best = float("inf")
    for _ in range(3):
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
        e1.synchronize()
        best = min(best, e0.elapsed_time(e1) * 1e-3 / reps / len(weights))
    del g
    return best


def run_breakdown(q, dev, peak):
    """GB/s per shape and M (default dispatch, static-weight plans): every M = 1..64 on the
    three 4-bit shapes, M in {4, 16, 64} on the mixed-precision ones."""
    from bit_quantized_gemm_qmm_b200.inputs import WORKLOADS
    out = {}
    tflops, _ = tensor_peak()
    for name in GATED + MIXED:
        wl = WORKLOADS[name]
        weights = make_weights(q, wl, dev)
        torch.cuda.synchronize()
        wbytes = wl.weight_bytes()
        Ms = range(1, 65) if name in GATED else MIXED_MS
        cells = {}
        for M in Ms:
            plan = default_plan(q, wl, M)
            t = time_cell(q, wl, weights, M, dev, plan)
            gbs = wbytes / t / 1e9
            bound = roofline_gbs(wl, M, peak, tflops)
            cells[str(M)] = {"gbs": round(gbs, 1), "us": round(t * 1e6, 3), "frac_of_measured": round(gbs / peak, 4),
                             "frac_of_nominal_8tbs": round(gbs / NOMINAL_HBM_GBS, 4),
                             "roofline_gbs": round(bound, 1), "frac_of_roofline": round(gbs / bound, 4),
                             "kernel": KERNEL_NAMES.get(plan.kernel, "?"), "plan": plan.as_dict()}
        g = [c["gbs"] for c in cells.values()]
        drops = [(int(a), round(1 - cells[b]["gbs"] / cells[a]["gbs"], 4)) for a, b in zip(list(cells)[:-1], list(cells)[1:])]
        worst = max(drops, key=lambda d: d[1]) if drops else (None, 0.0)
        out[name] = {"shape": f"K={wl.K} N={wl.N} {wl.bits}-bit g{wl.group} {str(wl.dtype).replace('torch.', '')}",
                     "weight_sets": len(weights), "weight_bytes_per_call": wbytes,
                     "min_frac_of_measured": round(min(g) / peak, 4), "mean_frac_of_measured": round(sum(g) / len(g) / peak, 4),
                     "largest_adjacent_drop": {"from_M": worst[0], "drop": worst[1]}, "M": cells}
        del weights
        torch.cuda.empty_cache()
        print(f"[breakdown] {name}: " + " ".join(f"{m}:{c['gbs']:.0f}" for m, c in cells.items()),
              file=sys.stderr, flush=True)
    return out


GROUPS = {  # one decoder layer's projections that share x (Qwen3-8B-like widths), 4-bit g64 fp16
    "qkv": {"K": 4096, "Ns": (4096, 1024, 1024), "sets": 18},
    "gate_up": {"K": 4096, "Ns": (14336, 14336), "sets": 4},
}
GROUP_MS = (1, 4, 16, 64)


NT_SHAPES = {  # the non-transposed form on the q/o and LM-head sizes: W' [K, N] quantized along N
    "qo_nt": {"K": 4096, "N": 4096, "dtype": torch.float16, "sets": 27},
    "lmhead_nt": {"K": 4096, "N": 151936, "dtype": torch.bfloat16, "sets": 1},
}
NT_MS = (1, 4, 16)


def run_nt(q, dev, peak):
    """GB/s of the non-transposed form (qmm_nt), 4-bit g64, per M; weight sets rotated
    (>= 2x L2), one CUDA graph of one call per set."""
    from bit_quantized_gemm_qmm_b200.inputs import w_input, x_input
    out = {}
    for name, c in NT_SHAPES.items():
        K, N, dt = c["K"], c["N"], c["dtype"]
        weights = []
        for i in range(c["sets"]):
            w = w_input(K, N, dt, i, 0.02 if dt is torch.bfloat16 else 1.0).to(dev)
            weights.append(q.quantize(w, 4, 64))
            del w
        wbytes = K * N // 2 + K * (N // 64) * 4
        cells = {}
        for M in NT_MS:
            x = x_input(M, K, dt).to(dev)
            y = torch.empty((M, N), dtype=dt, device=dev)
            for (P, S, B) in weights:
                q.qmm_nt(x, P, S, B, 4, 64, out=y)
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for (P, S, B) in weights:
                    q.qmm_nt(x, P, S, B, 4, 64, out=y)
            g.replay()
            torch.cuda.synchronize()
            reps = max(3, int(1e9 / (wbytes * len(weights))))
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(reps):
                g.replay()
            e1.record()
            e1.synchronize()
            t = e0.elapsed_time(e1) * 1e-3 / reps / len(weights)
            cells[str(M)] = {"gbs": round(wbytes / t / 1e9, 1), "us": round(t * 1e6, 3),
                             "frac_of_measured": round(wbytes / t / 1e9 / peak, 4)}
            del g
        out[name] = {"shape": f"W' [K={K}, N={N}] 4-bit g64 {str(dt).replace('torch.', '')}", "weight_sets": len(weights),
                     "kernel": "qmm_nta_kernel (CUDA cores, rows staged by cp.async)", "M": cells}
        del weights
        torch.cuda.empty_cache()
        print(f"[nt] {name}: " + " ".join(f"{m}:{v['gbs']:.0f}" for m, v in cells.items()), file=sys.stderr, flush=True)
    return out


def run_grouped(q, dev, peak):
    """One launch over a layer's matrices (qmm_grouped) against the same matrices as separate
    calls: GB/s of the group's weight bytes per M, weight sets rotated (>= 2x L2)."""
    from bit_quantized_gemm_qmm_b200.inputs import w_input, x_input
    out = {}
    stream = torch.cuda.current_stream(dev)
    for name, cfg in GROUPS.items():
        K, Ns = cfg["K"], cfg["Ns"]
        sets = []
        for i in range(cfg["sets"]):
            mats = []
            for j, N in enumerate(Ns):
                w = w_input(N, K, torch.float16, 500 + 10 * i + j, 1.0).to(dev)
                mats.append(q.quantize(w, 4, 64))
                del w
            sets.append(mats)
        torch.cuda.synchronize()
        gbytes = sum(N * K // 2 + N * (K // 64) * 4 for N in Ns)
        cells = {}
        for M in GROUP_MS:
            x = x_input(M, K, torch.float16).to(dev)
            outs = [torch.empty((M, N), dtype=torch.float16, device=dev) for N in Ns]
            plans = [q.plan_default(M, N, K, 4, 64, torch.float16) for N in Ns]
            for p_ in plans:
                p_.flags |= q.PLAN_STATIC_WEIGHTS
            gplan = q.make_plan(kernel=q.KERNEL_AUTO, flags=q.PLAN_PDL | q.PLAN_STATIC_WEIGHTS)

            def grouped():
                for mats in sets:
                    q.qmm_grouped(x, mats, 4, 64, outs=outs, plan=gplan)

            def separate():
                for mats in sets:
                    for (P, S, B), y, p_ in zip(mats, outs, plans):
                        q.qmm(x, P, S, B, 4, 64, out=y, plan=p_)

            res = {}
            for label, fn in (("grouped", grouped), ("separate", separate)):
                fn()
                torch.cuda.synchronize()
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    fn()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                best = float("inf")
                for _ in range(3):
                    g.replay()
                    torch.cuda.synchronize()
                    e0.record(stream)
                    for _ in range(10):
                        g.replay()
                    e1.record(stream)
                    e1.synchronize()
                    best = min(best, e0.elapsed_time(e1) * 1e-3 / 10 / len(sets))
                del g
                gbs = gbytes / best / 1e9
                res[label] = {"gbs": round(gbs, 1), "us": round(best * 1e6, 3), "frac_of_measured": round(gbs / peak, 4)}
            res["speedup"] = round(res["separate"]["us"] / res["grouped"]["us"], 3)
            cells[str(M)] = res
        out[name] = {"K": K, "Ns": list(Ns), "format": "4-bit g64 fp16", "weight_sets": len(sets),
                     "weight_bytes_per_group": gbytes, "M": cells}
        del sets
        torch.cuda.empty_cache()
        print(f"[grouped] {name}: " + " ".join(f"{m}:{c['grouped']['gbs']:.0f}/{c['separate']['gbs']:.0f}"
                                               for m, c in cells.items()), file=sys.stderr, flush=True)
    return out


def run_ours(args, rank, world):
    import bit_quantized_gemm_qmm_b200 as q
    dev = torch.device("cuda", torch.cuda.current_device())
    q.lib()  # loud failure if the CUDA library is missing
    wl, weights, xs, ys, plans = setup_workload(dev)
    wbytes = wl.weight_bytes()
    nsets = len(weights)
    calls_per_step = len(BENCH_MS) * nsets
    step_wbytes = wbytes * calls_per_step
    step_algo_bytes = sum((wbytes + 2 * M * wl.K + 2 * M * wl.N) * len(weights) for M in BENCH_MS)
    launches_per_step = sum(launches_per_call(q, wl, M, plans[M]) * len(weights) for M in BENCH_MS)

    def step(Ms=BENCH_MS):
        for M in Ms:
            x, y, p = xs[M], ys[M], plans[M]
            for (P, S, B) in weights:
                q.qmm(x, P, S, B, wl.bits, wl.group, out=y, plan=p)

    stream = torch.cuda.current_stream(dev)
    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for _ in range(max(3, args.warmup)):
        g.replay()
    torch.cuda.synchronize()

    # ---- clocks: sampled from a soak of the same replays right before the timed region
    # through to its end (the timed region alone is too short for a 200 ms sampler)
    clocks = ClockSampler(dev.index, not args.no_clocks)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if clocks.proc is not None:
        t_end = time.perf_counter() + CLOCK_SOAK_S
        while time.perf_counter() < t_end:
            for _ in range(20):
                g.replay()
            torch.cuda.synchronize()

    # ---- timed region: exactly K graph replays of the step
    barrier(world)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(args.steps):
        g.replay()
    e1.record(stream)
    e1.synchronize()
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    t_ms = max_over_ranks(e0.elapsed_time(e1), world)
    ms_per_step = t_ms / args.steps
    value = job_gbs(step_wbytes, ms_per_step, world)
    achieved = step_algo_bytes / (ms_per_step * 1e-3) / 1e9  # per GPU: the only kernels in the step

    # ---- eager figure (same calls, launched one by one)
    reps = max(5, args.steps // 4)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(reps):
        step()
    e1.record(stream)
    e1.synchronize()
    eager_ms = e0.elapsed_time(e1) / reps
    eager_value = step_wbytes / (eager_ms * 1e-3) / 1e9

    peak, peak_kind = measured_peaks()
    per_m = {}
    for M in BENCH_MS:
        t = time_cell(q, wl, weights, M, dev, plans[M])
        gbs = wbytes / t / 1e9
        per_m[f"M={M}"] = {"gbs": round(gbs, 1), "us_per_call": round(t * 1e6, 3),
                           "frac_of_measured": round(gbs / peak, 4), "frac_of_nominal_8tbs": round(gbs / NOMINAL_HBM_GBS, 4),
                           "plan": plans[M].as_dict()}

    # ---- end-to-end through the public API with host buffers
    e2e = run_e2e(wl, weights, plans, dev, max(5, args.steps // 10))
    del g
    torch.cuda.synchronize()
    breakdown = grouped = nt = None
    if not args.no_breakdown:
        del weights
        torch.cuda.empty_cache()
        breakdown = run_breakdown(q, dev, peak)
        grouped = run_grouped(q, dev, peak)
        nt = run_nt(q, dev, peak)

    kernel = KERNEL_NAMES.get(plans[BENCH_MS[0]].kernel, "?")
    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 6),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f16 (fp16 dequantized weights x fp16-converted bf16 activations, fp32 accumulation)",
        "data": "synthetic (seeded N(0,1) bf16 x, N(0,0.02^2) bf16 W, quantized by the library)",
        "config": {"workload": "lmhead: K=4096 N=151936 4-bit g64 bf16, M in {1,4,6,16}",
                   "weight_sets": nsets, "calls_per_step": calls_per_step,
                   "weight_bytes_per_call": wbytes,
                   "l2": f"one {wbytes / 1e6:.0f} MB weight matrix > 126 MB L2 (inputs larger than L2)",
                   "launch": "CUDA graph replay of the step", "eager_value_gbs": round(eager_value, 2),
                   "frac_of_nominal_8tbs": round(value / world / NOMINAL_HBM_GBS, 4), "per_M": per_m},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic_per_launch(),
                     "peak_kind": peak_kind, "kernel": kernel,
                     "algorithmic_bytes_per_launch": "weight bytes + 2*M*K (x) + 2*M*N (y), averaged over the "
                                                     "step's calls; time = step time / calls (launch gaps included)"},
        "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps,
    }
    if breakdown is not None:
        out["breakdown"] = breakdown
        out["grouped"] = grouped
        out["non_transposed"] = nt
    if clk:
        clk["window"] = f"{CLOCK_SOAK_S:.1f} s of the same replays immediately before the timed region, and the timed region"
        out["clocks"] = clk
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(wl, budget_s=12.0)
        out["cpu_baseline"]["single_thread"] = oracle_single_thread()
    if rank == 0:
        if args.breakdown_out:
            with open(args.breakdown_out, "w") as f:
                json.dump(out, f, indent=1)
        print(json.dumps(out), flush=True)


def run_e2e(wl, weights, plans, dev, steps):
    """Each step through the Python API: the step's inputs (x for each M, one pinned buffer, one
    copy) go from pinned host memory to the device, every call of the step runs, and every
    output comes back to pinned host memory before the step ends; the weights stay resident,
    as a model's do.  The output of one M goes back on a copy stream while the calls of the
    next M run, largest M first, so that only the smallest output's copy is left after the
    last call."""
    import bit_quantized_gemm_qmm_b200 as q
    from bit_quantized_gemm_qmm_b200.inputs import x_input
    S = len(weights)
    # the step's inputs (x of every M) in one pinned buffer, so one copy brings them over
    rows = sum(BENCH_MS)
    hx_all = torch.empty((rows, wl.K), dtype=wl.dtype).pin_memory()
    dx_all = torch.empty((rows, wl.K), dtype=wl.dtype, device=dev)
    hx, dx, r0 = {}, {}, 0
    for M in BENCH_MS:
        hx[M] = hx_all[r0:r0 + M]
        hx[M].copy_(x_input(M, wl.K, wl.dtype))
        dx[M] = dx_all[r0:r0 + M]
        r0 += M
    hy = {M: torch.empty((S, M, wl.N), dtype=wl.dtype).pin_memory() for M in BENCH_MS}
    dy = {M: torch.empty((S, M, wl.N), dtype=wl.dtype, device=dev) for M in BENCH_MS}
    outs = {M: list(dy[M].unbind(0)) for M in BENCH_MS}  # each call's own output slice
    stream = torch.cuda.current_stream(dev)
    copy_stream = torch.cuda.Stream(dev)
    done = {M: torch.cuda.Event() for M in BENCH_MS}

    def one_step():
        dx_all.copy_(hx_all, non_blocking=True)
        for M in sorted(BENCH_MS, reverse=True):
            for (P, S_, B), y in zip(weights, outs[M]):
                q.qmm(dx[M], P, S_, B, wl.bits, wl.group, out=y, plan=plans[M])
            done[M].record(stream)
            copy_stream.wait_event(done[M])
            with torch.cuda.stream(copy_stream):
                hy[M].copy_(dy[M], non_blocking=True)
        copy_stream.synchronize()
        stream.synchronize()

    one_step()
    t0 = time.perf_counter()
    for _ in range(steps):
        one_step()
    dt = (time.perf_counter() - t0) / steps
    h2d = sum(2 * M * wl.K for M in BENCH_MS)
    d2h = sum(2 * M * wl.N for M in BENCH_MS) * S
    value = wl.weight_bytes() * len(BENCH_MS) * S / dt / 1e9
    return {"value": round(value, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": round(dt * 1e3, 4), "api": "bit_quantized_gemm_qmm_b200.qmm (C ABI qmm_ex)",
            "calls_per_step": len(BENCH_MS) * S}


# The sources that decide the benchmark's launches: the kernels, the headers they are
# compiled from, and the dispatch that picks them and their plans.
TRAFFIC_SOURCES = ("qmm_api.cu", "qmm_common.cuh", "qmm_dq.cuh", "qmm_internal.h", "qmm_sk.cu", "qmm_stream.cu",
                   "sm100.cuh")


def traffic_per_launch():
    """DRAM bytes per launch from the committed ncu capture, if the sources of the profiled
    kernel and its dispatch still match the ones that were profiled (else null)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        d = json.load(open(path))
    except Exception:
        return None
    h = hashlib.sha256()
    for name in TRAFFIC_SOURCES:
        h.update(open(os.path.join(ROOT, "bit_quantized_gemm_qmm_b200", "csrc", name), "rb").read())
    if d.get("csrc_sha256") != h.hexdigest():
        return None
    return d.get("bytes_per_launch")


# ---------------------------------------------------------------------------- CPU oracle
def _oracle_inputs(wl, rows: int):
    """Oracle-quantized first `rows` rows of weight set 0 and the x of each M (numpy)."""
    import numpy as np

    import oracle
    from bit_quantized_gemm_qmm_b200.inputs import w_rows, x_input
    oracle.build()
    w = w_rows(wl.K, wl.dtype, 0, wl.w_sigma, 0, rows).view(torch.int16).numpy().view(np.uint16)
    pq = oracle.quantize(w, wl.bits, wl.group, wl.dtype == torch.bfloat16)
    xs = {M: x_input(M, wl.K, wl.dtype).view(torch.int16).numpy().view(np.uint16) for M in BENCH_MS}
    return pq, xs


def _oracle_pass(wl, pq, xs, rows: int) -> float:
    import oracle
    p, s, b = pq
    t0 = time.perf_counter()
    for M in BENCH_MS:
        oracle.qmm(xs[M], p[:rows], s[:rows], b[:rows], wl.K, wl.bits, wl.group, wl.dtype == torch.bfloat16)
    return time.perf_counter() - t0


def oracle_single_thread():
    """Seconds of one oracle call on one host thread (a separate process with OMP_NUM_THREADS=1),
    at M = 4 on the tiny and the q/o configurations, whole matrices."""
    import subprocess
    code = (
        "import json, time, sys\n"
        "sys.path.insert(0, %r)\n"
        "import torch, oracle\n"
        "from bit_quantized_gemm_qmm_b200.inputs import WORKLOADS, w_input, x_input\n"
        "from bench import _oracle_inputs\n"
        "oracle.build()\n"
        "out = {}\n"
        "for name in ('tiny', 'qo'):\n"
        "    wl = WORKLOADS[name]\n"
        "    (p, s, b), xs = _oracle_inputs(wl, wl.N)\n"
        "    x = xs[4]\n"
        "    t0 = time.perf_counter()\n"
        "    oracle.qmm(x, p, s, b, wl.K, wl.bits, wl.group, wl.dtype == torch.bfloat16)\n"
        "    out[name + '_m4_s'] = round(time.perf_counter() - t0, 4)\n"
        "print(json.dumps(out))\n") % ROOT
    env = dict(os.environ, OMP_NUM_THREADS="1")
    try:
        r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, env=env, cwd=ROOT, timeout=600)
        return json.loads(r.stdout.strip().splitlines()[-1])
    except Exception as e:  # reported, never fatal: the single-thread time is context only
        return {"error": str(e)[:200]}


def cpu_baseline(wl, budget_s: float = 12.0, rows: int = 8192):
    """The CPU oracle as it stands, on the host cores: one call per M on the first `rows` rows
    of the weight matrix, repeated for about `budget_s` seconds; GB/s counts the weight bytes
    of those rows."""
    cores = int(os.environ.get("OMP_NUM_THREADS", host_cores()))
    rows = min(rows, wl.N)
    pq, xs = _oracle_inputs(wl, rows)
    t_total, passes = 0.0, 0
    while passes == 0 or t_total < budget_s:
        t_total += _oracle_pass(wl, pq, xs, rows)
        passes += 1
    nbytes = passes * len(BENCH_MS) * wl.weight_bytes() * rows / wl.N
    return {"value": round(nbytes / t_total / 1e9, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{passes} pass(es) of one call per M in {list(BENCH_MS)} on rows 0..{rows - 1} of the "
                      f"{wl.N}-row weight matrix ({t_total:.1f} s)"}


def run_reference(args, rank, world):
    """Reference arm: the CPU oracle, as it stands, on the same workload, metric and unit.
    Each step is one call per M on a row sample of weight set 0, sized so that all steps
    take about two minutes."""
    if rank != 0:
        return
    from bit_quantized_gemm_qmm_b200.inputs import WORKLOADS
    wl = WORKLOADS[WORKLOAD]
    cores = int(os.environ.get("OMP_NUM_THREADS", host_cores()))
    probe = min(wl.N, 4096)
    pq, xs = _oracle_inputs(wl, probe)
    t_probe = _oracle_pass(wl, pq, xs, probe)
    rows = int(min(probe, max(64, probe * (120.0 / max(1, args.steps + args.warmup)) / max(t_probe, 1e-6))))
    for _ in range(args.warmup):
        _oracle_pass(wl, pq, xs, rows)
    t_total = 0.0
    for _ in range(args.steps):
        t_total += _oracle_pass(wl, pq, xs, rows)
    row_bytes = wl.weight_bytes() / wl.N
    value = round(args.steps * len(BENCH_MS) * rows * row_bytes / t_total / 1e9, 4)
    sample = f"{rows} of {wl.N} rows of weight set 0, one call per M in {list(BENCH_MS)} per step"
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(t_total * 1e3 / max(1, args.steps), 3),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)",
           "data": "synthetic (seeded N(0,1) bf16 x, N(0,0.02^2) bf16 W)",
           "config": {"workload": "lmhead: K=4096 N=151936 4-bit g64 bf16, M in {1,4,6,16}"},
           "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": sample},
           "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def _parse_ms(spec: str):
    out = []
    for part in spec.split(","):
        if "-" in part:
            a, b = part.split("-")
            out.extend(range(int(a), int(b) + 1))
        elif part:
            out.append(int(part))
    return out


def run_sweep(args):
    """GB/s per (configuration, M): one CUDA graph of one call per rotated weight set,
    replayed; per-call time = graph time / sets."""
    import bit_quantized_gemm_qmm_b200 as q
    from bit_quantized_gemm_qmm_b200.inputs import WORKLOADS, w_input, x_input
    dev = torch.device("cuda", torch.cuda.current_device())
    peak, peak_kind = measured_peaks()
    results = {"peak_gbs": peak, "peak_kind": peak_kind, "configs": {}}
    stream = torch.cuda.current_stream(dev)
    for name in args.sweep_configs.split(","):
        wl = WORKLOADS[name]
        weights = []
        for i in range(wl.sets):
            w = w_input(wl.N, wl.K, wl.dtype, i, wl.w_sigma).to(dev)
            weights.append(q.quantize(w, wl.bits, wl.group))
            del w
        torch.cuda.synchronize()
        wbytes = wl.weight_bytes()
        rows = {}
        for M in _parse_ms(args.sweep_ms):
            x = x_input(M, wl.K, wl.dtype).to(dev)
            y = torch.empty((M, wl.N), dtype=wl.dtype, device=dev)
            if args.sweep_plan:
                f = [int(v) for v in args.sweep_plan.split(":")]
                kern, split, warps = f[:3]
                flags = f[3] if len(f) > 3 else q.PLAN_PDL | q.PLAN_STATIC_WEIGHTS
                plan = q.make_plan(kernel=kern, split=split, warps=warps, flags=flags)
            else:
                plan = q.plan_default(M, wl.N, wl.K, wl.bits, wl.group, wl.dtype)
                plan.flags |= q.PLAN_STATIC_WEIGHTS
            for (P, S, B) in weights:
                q.qmm(x, P, S, B, wl.bits, wl.group, out=y, plan=plan)
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for (P, S, B) in weights:
                    q.qmm(x, P, S, B, wl.bits, wl.group, out=y, plan=plan)
            reps = max(3, int(2e9 / (wbytes * len(weights))))  # ~2 GB streamed per timing
            for _ in range(3):
                g.replay()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            best = float("inf")
            for _ in range(3):
                torch.cuda.synchronize()
                e0.record(stream)
                for _ in range(reps):
                    g.replay()
                e1.record(stream)
                e1.synchronize()
                best = min(best, e0.elapsed_time(e1) / reps / len(weights))
            gbs = wbytes / (best * 1e-3) / 1e9
            rows[M] = {"gbs": round(gbs, 1), "us": round(best * 1e3, 3), "frac": round(gbs / peak, 4),
                       "frac_nominal": round(gbs / NOMINAL_HBM_GBS, 4), "plan": plan.as_dict()}
            del g
        results["configs"][name] = {"N": wl.N, "K": wl.K, "bits": wl.bits, "group": wl.group,
                                    "dtype": str(wl.dtype), "sets": wl.sets, "weight_bytes": wbytes,
                                    "M": rows}
        del weights
        torch.cuda.empty_cache()
        print(f"[sweep] {name}: " + " ".join(f"{m}:{r['gbs']:.0f}" for m, r in rows.items()),
              file=sys.stderr, flush=True)
    with open(args.sweep, "w") as f:
        json.dump(results, f, indent=1)


def main():
    args = parse()
    rank, world = init_dist(args)
    try:
        if args.sweep:
            run_sweep(args)
        elif args.impl == "reference":
            run_reference(args, rank, world)
        else:
            run_ours(args, rank, world)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
