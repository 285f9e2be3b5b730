#!/usr/bin/env python3
"""Benchmark of the batch-1 Q4 GEMV decode stream on B200.

Workload (one "step"): batch-1 GEMV y = W_hat x over the 4096x11008 weight
shape in both Q4 formats and both orientations -- Q4_0 and super-block (ksb)
weights, M=4096 x K=11008 and M=11008 x K=4096 -- each over ``--copies``
distinct copies of its packed matrix, launched back to back (CUDA graph,
programmatic dependent launch).  A step streams ~1.6 GB of packed weights,
far more than the 126 MB L2, so every GEMV reads cold weights.

Metric: streamed-weight GB/s = packed weight bytes / device time.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--suite FILE]

With N > 1 (torchrun), every rank runs the same workload on its own GPU
(independent replicas: the path has no exchange step) and rank 0 prints the
aggregate over ranks with the max of the per-rank device times.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Q4 GEMV streamed-weight GB/s and % of HBM peak (4096x11008, batch 1)"
CASES = [("q4_0", 4096, 11008), ("q4_0", 11008, 4096), ("ksb", 4096, 11008), ("ksb", 11008, 4096)]
FALLBACK_HBM_GBS = 6650.0

# DRAM bytes (read + write) of one GEMV launch, the q4_0 4096x11008 case, from
# one ncu capture (profiles/gemv_q4_0_4096x11008.md).  Reported only while the
# GEMV sources hash to what was profiled; any change to the kernel makes it null.
GEMV_TRAFFIC = {
    "bytes": 25406976,
    "sources": {
        "bit_gemv_q4_b200/csrc/gq_gemv.cu": "2097710892fc724426aeafb75a26e0e3488edc2a224265dbdbaa265152e66880",
        "bit_gemv_q4_b200/csrc/gq_device.cuh": "8eec6074ffd6e2337bf1ea2999f16285b22b3bca681a3cbf9c4acd0b821173c2",
    },
}


def gemv_traffic():
    import hashlib
    for rel, digest in GEMV_TRAFFIC["sources"].items():
        try:
            with open(os.path.join(ROOT, rel), "rb") as f:
                if hashlib.sha256(f.read()).hexdigest() != digest:
                    return None
        except OSError:
            return None
    return GEMV_TRAFFIC["bytes"]


def packed_bytes(fmt, M, K):
    return M * (K // 32 * 18 if fmt == "q4_0" else K // 256 * 138)


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ----------------------------------------------------------------- clocks
THROTTLE_BITS = {  # nvidia-smi clocks_event_reasons bit -> name
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
    0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
    0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
    0x100: "display_clock_setting",
}


class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons while running."""

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu),
                 "--query-gpu=clocks.sm,clocks.max.sm,clocks_event_reasons.active",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.t.join(timeout=2)

    def summary(self):
        sm, mx, reasons = [], [], set()
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 3:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
                bits = int(parts[2], 16)
            except ValueError:
                continue
            for b, name in THROTTLE_BITS.items():
                if bits & b and name != "gpu_idle":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------- distributed
def dist_setup():
    import torch
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return rank, ws, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, ws: int) -> float:
    """Max of a per-rank scalar (device time) over all ranks."""
    if ws == 1:
        return v
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(units_per_rank: float, ms_per_rank: float, ws: int) -> tuple[float, float]:
    """(whole-job units per second, max ms over ranks): units of all ranks
    over the slowest rank's device time."""
    ms = max_over_ranks(ms_per_rank, ws)
    return units_per_rank * ws / (ms / 1e3), ms


# --------------------------------------------------------------- our arm
def build_gemv_set(gq, synth, copies, device, pdl=True):
    """Packed weight copies, activations and outputs for the four cases."""
    import torch
    sets = []
    for ci, (fmt, M, K) in enumerate(CASES):
        w = synth.gaussian_weights(M, K, seed=100 + ci, device=device)
        quant = gq.gq_quantize_q4_0 if fmt == "q4_0" else gq.gq_quantize_ksb
        q = quant(w.view(-1))
        del w
        nb = packed_bytes(fmt, M, K)
        Wc = torch.empty((copies, nb), dtype=torch.uint8, device=device)
        Wc.copy_(q.view(1, nb).expand(copies, nb))
        x = synth.activations(1, K, seed=200 + ci, dtype=torch.float16, device=device)
        y = torch.empty((1, M), dtype=torch.float16, device=device)
        gemv = gq.gq_gemv_q4_0 if fmt == "q4_0" else gq.gq_gemv_ksb
        sets.append(dict(fmt=fmt, M=M, K=K, W=Wc, x=x, y=y, gemv=gemv, nbytes=nb, ws=None,
                         kernels=1))
    torch.cuda.synchronize()
    return sets


def gemv_workspace(gq, fmt, M, K, B, xdtype, device):
    """A zeroed workspace for gq_gemv_* (None when the case needs none).  The
    calls of one stream run in order, so they could share one."""
    import torch
    code = gq.GQ_FMT_Q4_0 if fmt == "q4_0" else gq.GQ_FMT_KSB
    need = gq.gq_gemv_workspace_bytes(code, M, K, B, xdtype)
    return torch.zeros(need, dtype=torch.uint8, device=device) if need else None


def launch_case(gq, s, copies, flags):
    for c in range(copies):
        s["gemv"](s["W"][c], s["M"], s["K"], s["x"], y_dtype=s["y"].dtype, out=s["y"], flags=flags,
                  workspace=s["ws"])


def capture(fn):
    import torch
    fn()  # eager warm-up outside capture (sets kernel attributes)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


def time_graph(g, steps, warmup, ws):
    import torch
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    barrier(ws)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    barrier(ws)
    return e0.elapsed_time(e1)


def run_ours(args, rank, ws, local):
    import torch
    import bit_gemv_q4_b200 as gq
    import synth

    dev = torch.device("cuda", torch.cuda.current_device())
    copies = args.copies
    sets = build_gemv_set(gq, synth, copies, dev)
    flags = gq.GQ_GEMV_PDL
    wbytes_step = sum(s["nbytes"] for s in sets) * copies
    algo_bytes_step = sum(s["nbytes"] + s["K"] * 2 + s["M"] * 2 for s in sets) * copies
    launches_step = sum(s["kernels"] for s in sets) * copies

    def step():
        for s in sets:
            launch_case(gq, s, copies, flags)

    g = capture(step)
    with ClockSampler(local) as clk:
        ms = time_graph(g, args.steps, args.warmup, ws)
    gbs, ms_max = aggregate(wbytes_step * args.steps / 1e9, ms, ws)
    ms_per_step = ms_max / args.steps
    launches = launches_step * args.steps

    # per-case breakdown (same kernel, each case timed alone)
    cases = {}
    case_steps = max(20, args.steps // 10)
    for s in sets:
        gc = capture(lambda s=s: launch_case(gq, s, copies, flags))
        mc = time_graph(gc, case_steps, args.warmup, ws)
        us = mc * 1e3 / (case_steps * copies)
        cases[f"{s['fmt']} M={s['M']} K={s['K']}"] = {
            "gbs": round(s["nbytes"] / (us * 1e-6) / 1e9, 1), "us_per_gemv": round(us, 3)}
        del gc
    # same stream without programmatic dependent launch, for contrast
    g_nopdl = capture(lambda: [launch_case(gq, s, copies, 0) for s in sets])
    ms_nopdl = time_graph(g_nopdl, max(20, args.steps // 10), args.warmup, ws)
    nopdl_gbs = wbytes_step * max(20, args.steps // 10) / (ms_nopdl / 1e3) / 1e9
    del g_nopdl

    # practical ceiling: the same weight copies read once each by a plain
    # streaming-read kernel (gq_stream_read), one launch per matrix, same graph
    sink = torch.zeros(1, dtype=torch.int32, device=dev)
    g_read = capture(lambda: [gq.gq_stream_read(s["W"][c], sink) for s in sets
                              for c in range(copies)])
    read_steps = max(20, args.steps // 10)
    ms_read = time_graph(g_read, read_steps, args.warmup, ws)
    read_gbs = wbytes_step * read_steps / (ms_read / 1e3) / 1e9
    del g_read

    # end to end through the public API with host buffers: each step copies
    # the four activation vectors from pinned host memory, runs the step's
    # GEMVs and reads the four results back into pinned host memory
    hx = [s["x"].cpu().pin_memory() for s in sets]
    hy = [torch.empty(s["y"].shape, dtype=s["y"].dtype).pin_memory() for s in sets]

    def e2e_step():
        for i, s in enumerate(sets):
            s["x"].copy_(hx[i], non_blocking=True)
        for s in sets:
            launch_case(gq, s, copies, flags)
        for i, s in enumerate(sets):
            hy[i].copy_(s["y"], non_blocking=True)

    e2e_steps = max(20, args.steps // 10)
    try:
        ge = capture(e2e_step)
        ms_e2e = time_graph(ge, e2e_steps, args.warmup, ws)
        e2e_mode = "CUDA graph with host copies"
        del ge
    except Exception:  # capture of pageable/pinned copies unsupported: eager
        for _ in range(args.warmup):
            e2e_step()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(e2e_steps):
            e2e_step()
        e1.record()
        torch.cuda.synchronize()
        ms_e2e = e0.elapsed_time(e1)
        e2e_mode = "eager launches with host copies"
    e2e_gbs, _ = aggregate(wbytes_step * e2e_steps / 1e9, ms_e2e, ws)
    h2d = sum(s["K"] * 2 for s in sets)
    d2h = sum(s["M"] * 2 for s in sets)
    del g

    peak, peak_src = measured_peaks()
    per_gpu_algo_gbs = algo_bytes_step / (ms_per_step * 1e-3) / 1e9
    result = {
        "metric": METRIC, "value": round(gbs, 1), "unit": "GB/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f16", "data": "synthetic",
        "config": {
            "workload": ("batch-1 GEMV, Q4_0 and super-block weights, 4096x11008 in both "
                         "orientations (M=4096 K=11008 and M=11008 K=4096), x fp16, y fp16, "
                         f"{copies} copies of each matrix per step"),
            "weights_per_step_bytes": wbytes_step,
            "l2": "inputs larger than L2 (weights rotated over %.2f GB per step)" % (wbytes_step / 1e9),
            "launch": "CUDA graph, programmatic dependent launch",
            "parallelism": "replicas" if ws > 1 else "single GPU",
        },
        "frac_of_peak": round(gbs / ws / peak, 4),
        "frac_of_nominal_8tbs": round(gbs / ws / 8000.0, 4),
        "roofline": {"bound": "hbm", "achieved": round(per_gpu_algo_gbs, 1), "peak": peak,
                     "peak_source": f"{peak_src} hbm_gbs", "unit": "GB/s",
                     "frac": round(per_gpu_algo_gbs / peak, 4), "traffic": gemv_traffic(),
                     "kernel": "gemv_kernel (all four cases)"},
        "cases": cases,
        "no_pdl_gbs": round(nopdl_gbs, 1),
        "read_ceiling": {"gbs": round(read_gbs, 1), "frac_of_peak": round(read_gbs / peak, 4),
                         "value_frac_of_ceiling": round(gbs / ws / read_gbs, 4),
                         "what": "the same weight copies, one plain streaming-read launch "
                                 "(gq_stream_read) per matrix, same CUDA graph"},
        "e2e": {"value": round(e2e_gbs, 1), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "mode": e2e_mode},
        "gpu_launches": launches,
        "clocks": clk.summary(),
    }
    return result


# ---------------------------------------------------- the oracle on the host
class OracleSample:
    """The four cases (one matrix each), quantized by the oracle; ``run``
    times the oracle's product over them on the host cores."""

    def __init__(self):
        import oracle
        import synth
        import torch
        oracle.build()
        self.oracle = oracle
        self.mats = []
        for ci, (fmt, M, K) in enumerate(CASES):
            w = synth.gaussian_weights(M, K, seed=100 + ci)
            f = oracle.FMT_Q4_0 if fmt == "q4_0" else oracle.FMT_KSB
            q, _ = oracle.quantize(f, w.numpy().ravel())
            x = synth.activations(1, K, seed=200 + ci, dtype=torch.float16).numpy()
            self.mats.append((f, q, M, K, x, packed_bytes(fmt, M, K)))

    def run(self, seconds: float):
        """Whole passes over the four cases until `seconds` have passed;
        returns (GB/s of packed weights, threads, description)."""
        done, nbytes, t0 = 0, 0, time.perf_counter()
        while True:
            f, q, M, K, x, nb = self.mats[done % len(self.mats)]
            self.oracle.gemm(f, q, M, K, x)
            done += 1
            nbytes += nb
            el = time.perf_counter() - t0
            if el >= seconds and done % len(self.mats) == 0:
                break
        desc = (f"{done} oracle GEMVs ({done // len(self.mats)} pass(es) over the four cases, "
                f"one matrix each) in {el:.1f} s")
        return nbytes / el / 1e9, self.oracle.num_threads(), desc


def run_reference(args, rank, ws):
    """The oracle as it stands, on this host's cores, same metric and config;
    each step is one pass over the four cases."""
    if rank != 0:
        return None
    smp = OracleSample()
    for _ in range(args.warmup):
        smp.run(0.0)
    vals, t0 = [], time.perf_counter()
    cores = smp.oracle.num_threads()
    for _ in range(args.steps):
        v, cores, _ = smp.run(0.0)
        vals.append(v)
    el = time.perf_counter() - t0
    value = statistics.median(vals)
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "GB/s",
        "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(el * 1e3 / max(1, args.steps), 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": ("batch-1 GEMV, Q4_0 and super-block weights, 4096x11008 in "
                                "both orientations, x fp16; one matrix per case per step")},
        "cpu_baseline": {"value": round(value, 3), "unit": "GB/s", "cores": cores,
                         "kind": "oracle",
                         "sample": f"{args.steps} steps, each one oracle GEMV of each case"},
        "e2e": {"value": round(value, 3), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


# ------------------------------------------------------------------ suite
def _timed(fn, reps, warmup=3):
    """Device ms per call of fn(), CUDA events on the current stream."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def _graph_ms_per_launch(fn, launches, reps):
    g = capture(fn)
    ms = _timed(g.replay, reps)
    del g
    return ms / launches


def run_suite(path):
    """Every row of the hot path on its own workload; one JSON line per row."""
    import torch
    import bit_gemv_q4_b200 as gq
    import synth
    dev = torch.device("cuda", torch.cuda.current_device())
    peak, peak_src = measured_peaks()
    out = open(path, "w")

    def emit(d):
        out.write(json.dumps(d) + "\n")
        out.flush()
        print("suite:", json.dumps(d), file=sys.stderr, flush=True)

    def quant(fmt, w):
        return (gq.gq_quantize_q4_0 if fmt == "q4_0" else gq.gq_quantize_ksb)(w.view(-1))

    # --- single GEMVs (decode shapes), cold weights, graph + PDL
    for fmt, M, K, B, xdt, ydt, name, use_ws in (
            ("q4_0", 256, 1024, 1, torch.float32, torch.float32, "tiny 256x1024 fp32", False),
            ("q4_0", 4096, 4096, 1, torch.float16, torch.float16, "decode 4096x4096", False),
            ("ksb", 11008, 4096, 1, torch.float16, torch.float16, "MLP 11008x4096 ksb B=1", False),
            ("ksb", 11008, 4096, 8, torch.float16, torch.float16, "MLP 11008x4096 ksb B=8", False),
            ("q4_0", 11008, 4096, 8, torch.float16, torch.float16, "MLP 11008x4096 q4_0 B=8", False),
            # the batch-1 integer tensor-core path (workspace given), for comparison
            ("q4_0", 4096, 4096, 1, torch.float16, torch.float16, "decode 4096x4096, integer path", True),
            ("q4_0", 4096, 11008, 1, torch.float16, torch.float16, "4096x11008, integer path", True),
            ("q4_0", 11008, 4096, 1, torch.float16, torch.float16, "11008x4096, integer path", True)):
        w = synth.gaussian_weights(M, K, seed=7, device=dev)
        q = quant(fmt, w)
        del w
        nb = q.numel()
        copies = max(4, int(512e6 // nb))
        Wc = torch.empty((copies, nb), dtype=torch.uint8, device=dev)
        Wc.copy_(q.view(1, nb).expand(copies, nb))
        x = synth.activations(B, K, seed=8, dtype=xdt, device=dev)
        y = torch.empty((B, M), dtype=ydt, device=dev)
        f = gq.gq_gemv_q4_0 if fmt == "q4_0" else gq.gq_gemv_ksb
        wsp = gemv_workspace(gq, fmt, M, K, B, xdt, dev) if use_ws else None
        ms = _graph_ms_per_launch(
            lambda: [f(Wc[i], M, K, x, y_dtype=ydt, out=y, flags=gq.GQ_GEMV_PDL, workspace=wsp)
                     for i in range(copies)],
            copies, 20)
        emit({"row": "gemv", "workload": name, "format": fmt, "M": M, "K": K, "B": B,
              "us": round(ms * 1e3, 3), "weight_gbs": round(nb / (ms * 1e-3) / 1e9, 1),
              "frac_of_peak": round(nb / (ms * 1e-3) / 1e9 / peak, 4),
              "gflops": round(2 * M * K * B / (ms * 1e-3) / 1e9, 1)})
        del Wc

    # --- read ceiling of one launch: the same rotated copies of each headline
    # matrix read once by a plain streaming-read kernel, graph of launches
    sink = torch.zeros(1, dtype=torch.int32, device=dev)
    for fmt, M, K in CASES:
        nb = packed_bytes(fmt, M, K)
        copies = max(4, int(512e6 // nb))
        buf = torch.empty((copies, nb), dtype=torch.uint8, device=dev)
        buf.fill_(7)
        ms = _graph_ms_per_launch(lambda: [gq.gq_stream_read(buf[i], sink) for i in range(copies)],
                                  copies, 20)
        emit({"row": "read_ceiling", "workload": f"plain streaming read of one {fmt} {M}x{K} "
              "matrix per launch", "bytes": nb, "us": round(ms * 1e3, 3),
              "gbs": round(nb / (ms * 1e-3) / 1e9, 1),
              "frac_of_peak": round(nb / (ms * 1e-3) / 1e9 / peak, 4)})
        del buf

    # --- whole-model weight stream: 32 layers x (4 x 4096^2 + 3 x 11008x4096)
    for fmt in ("q4_0", "ksb"):
        shapes = []
        for layer in range(32):
            shapes += [(4096, 4096)] * 4 + [(11008, 4096)] * 3
        mats, total = [], 0
        for i, (M, K) in enumerate(shapes):
            w = synth.gaussian_weights(M, K, seed=30000 + i, device=dev)
            mats.append((quant(fmt, w), M, K))
            total += mats[-1][0].numel()
            del w
        x = synth.activations(1, 4096, seed=9, dtype=torch.float16, device=dev)
        ys = {M: torch.empty((1, M), dtype=torch.float16, device=dev) for M in (4096, 11008)}
        f = gq.gq_gemv_q4_0 if fmt == "q4_0" else gq.gq_gemv_ksb
        wss = {M: None for M in (4096, 11008)}
        ms = _graph_ms_per_launch(
            lambda: [f(qm, M, K, x, out=ys[M], flags=gq.GQ_GEMV_PDL, workspace=wss[M])
                     for qm, M, K in mats], 1, 5)
        emit({"row": "model_stream", "workload": "32 layers x (4 x 4096x4096 + 3 x 11008x4096), "
              "224 batch-1 GEMVs, one CUDA graph", "format": fmt, "weight_bytes": total,
              "ms": round(ms, 3), "weight_gbs": round(total / (ms * 1e-3) / 1e9, 1),
              "frac_of_peak": round(total / (ms * 1e-3) / 1e9 / peak, 4),
              "matrices_per_s": round(224 / (ms * 1e-3), 1)})
        # the same 224 products as one grouped call (one launch, x loaded once per CTA)
        fg = gq.gq_gemv_q4_0_grouped if fmt == "q4_0" else gq.gq_gemv_ksb_grouped
        outs = [torch.empty((1, M), dtype=torch.float16, device=dev) for _, M, _ in mats]
        Ws, Ms = [m[0] for m in mats], [m[1] for m in mats]
        ms = _graph_ms_per_launch(
            lambda: fg(Ws, Ms, 4096, x, outs=outs, flags=gq.GQ_GEMV_PDL), 1, 5)
        emit({"row": "model_stream_grouped", "workload": "32 layers x (4 x 4096x4096 + 3 x "
              "11008x4096), 224 batch-1 GEMVs in one grouped call", "format": fmt,
              "weight_bytes": total, "ms": round(ms, 3),
              "weight_gbs": round(total / (ms * 1e-3) / 1e9, 1),
              "frac_of_peak": round(total / (ms * 1e-3) / 1e9 / peak, 4),
              "matrices_per_s": round(224 / (ms * 1e-3), 1)})
        del Ws, outs
        del mats
        torch.cuda.empty_cache()

    # --- tensor-core dequant-GEMM, W 11008x4096, X bf16 [B, 4096]
    M, K = 11008, 4096
    for fmt in ("q4_0", "ksb"):
        w = synth.gaussian_weights(M, K, seed=11, device=dev)
        q = quant(fmt, w)
        del w
        nb = q.numel()
        copies = 6
        Wc = torch.empty((copies, nb), dtype=torch.uint8, device=dev)
        Wc.copy_(q.view(1, nb).expand(copies, nb))
        f = gq.gq_gemm_q4_0 if fmt == "q4_0" else gq.gq_gemm_ksb
        for B in (16, 64, 256):
            X = synth.activations(B, K, seed=12, dtype=torch.bfloat16, device=dev)
            Y = torch.empty((B, M), dtype=torch.float32, device=dev)
            # one zeroed workspace for every call: a call leaves it ready for the next
            code = gq.GQ_FMT_Q4_0 if fmt == "q4_0" else gq.GQ_FMT_KSB
            wsp = torch.zeros(max(gq.gq_gemm_workspace_bytes(code, M, K, B), 1), dtype=torch.uint8,
                              device=dev)
            ms = _graph_ms_per_launch(
                lambda: [f(Wc[i], M, K, X, out=Y, workspace=wsp) for i in range(copies)], copies, 10)
            tf = 2.0 * M * K * B / (ms * 1e-3) / 1e12
            emit({"row": "gemm", "workload": f"W {M}x{K} x X bf16 [{B},{K}], Y fp32",
                  "format": fmt, "B": B, "us": round(ms * 1e3, 2), "tflops": round(tf, 1),
                  "weight_gbs": round(nb / (ms * 1e-3) / 1e9, 1),
                  "frac_of_bf16_peak": round(tf / 1615.2, 4),
                  "note": "useful flops 2*M*K*B; the exact hi/lo split issues twice that"})
        del Wc

    # --- quantize and dequantize 1e9 weights ~ N(0, 0.02^2)
    n = 1_000_000_000
    w = synth.gaussian_weights(n // 8000, 8000, seed=4, frac=0.0, device=dev).view(-1)
    for fmt, nbytes in (("q4_0", n // 32 * 18), ("ksb", n // 256 * 138)):
        q = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        fq = gq.gq_quantize_q4_0 if fmt == "q4_0" else gq.gq_quantize_ksb
        ms = _timed(lambda: fq(w, out=q), 5)
        emit({"row": "quantize", "workload": "1e9 fp32 weights", "format": fmt,
              "ms": round(ms, 3), "gweights_per_s": round(n / (ms * 1e-3) / 1e9, 2),
              "gbs": round((4 * n + nbytes) / (ms * 1e-3) / 1e9, 1),
              "frac_of_peak": round((4 * n + nbytes) / (ms * 1e-3) / 1e9 / peak, 4)})
        fd = gq.gq_dequantize_q4_0 if fmt == "q4_0" else gq.gq_dequantize_ksb
        ms = _timed(lambda: fd(q, n, out=w), 5)
        emit({"row": "dequantize", "workload": "1e9 weights to fp32", "format": fmt,
              "ms": round(ms, 3), "gweights_per_s": round(n / (ms * 1e-3) / 1e9, 2),
              "gbs": round((4 * n + nbytes) / (ms * 1e-3) / 1e9, 1),
              "frac_of_peak": round((4 * n + nbytes) / (ms * 1e-3) / 1e9 / peak, 4)})
        del q
    out.close()


def run_single(spec, launches, batch, flags, use_ws=False):
    """A few launches of one hot-path call (for profilers).  spec:
    "gemv:q4_0:4096:11008" / "gemm:ksb:11008:4096" (distinct copies of one
    matrix), "grouped:q4_0:<layers>" (the decoder-layer matrices
    4 x 4096x4096 + 3 x 11008x4096 per layer in one grouped call), or
    "quantize:ksb:<n>" / "dequantize:q4_0:<n>" (n weights)."""
    import torch
    import bit_gemv_q4_b200 as gq
    import synth
    dev = torch.device("cuda", torch.cuda.current_device())
    parts = spec.split(":")
    if parts[0] == "grouped":
        fmt, layers = parts[1], int(parts[2])
        quant = gq.gq_quantize_q4_0 if fmt == "q4_0" else gq.gq_quantize_ksb
        Ms = ([4096] * 4 + [11008] * 3) * layers
        Ws, nb = [], 0
        for i, M in enumerate(Ms):
            w = synth.gaussian_weights(M, 4096, seed=30000 + i, device=dev)
            Ws.append(quant(w.view(-1)))
            nb += Ws[-1].numel()
            del w
        x = synth.activations(batch, 4096, seed=9, dtype=torch.float16, device=dev)
        outs = [torch.empty((batch, M), dtype=torch.float16, device=dev) for M in Ms]
        fg = gq.gq_gemv_q4_0_grouped if fmt == "q4_0" else gq.gq_gemv_ksb_grouped
        for _ in range(launches):
            fg(Ws, Ms, 4096, x, outs=outs, flags=flags)
        torch.cuda.synchronize()
        print(json.dumps({"single": spec, "batch": batch, "launches": launches, "bytes": nb}))
        return
    if parts[0] in ("quantize", "dequantize"):
        fmt, n = parts[1], int(parts[2])
        x = torch.randn(n, device=dev, dtype=torch.float32)
        qf = gq.gq_quantize_q4_0 if fmt == "q4_0" else gq.gq_quantize_ksb
        q = qf(x)
        for _ in range(launches):
            if parts[0] == "quantize":
                qf(x, out=q)
            else:
                (gq.gq_dequantize_q4_0 if fmt == "q4_0" else gq.gq_dequantize_ksb)(q, n, out=x)
        torch.cuda.synchronize()
        print(json.dumps({"single": spec, "launches": launches, "bytes": q.numel() + 4 * n}))
        return
    kind, fmt, M, K = parts
    M, K = int(M), int(K)
    w = synth.gaussian_weights(M, K, seed=1, device=dev)
    q = (gq.gq_quantize_q4_0 if fmt == "q4_0" else gq.gq_quantize_ksb)(w.view(-1))
    del w
    nb = q.numel()
    copies = 6
    Wc = torch.empty((copies, nb), dtype=torch.uint8, device=dev)
    Wc.copy_(q.view(1, nb).expand(copies, nb))
    if kind == "gemv":
        x = synth.activations(batch, K, seed=2, dtype=torch.float16, device=dev)
        f = gq.gq_gemv_q4_0 if fmt == "q4_0" else gq.gq_gemv_ksb
        y = torch.empty((batch, M), dtype=torch.float16, device=dev)
        wsp = gemv_workspace(gq, fmt, M, K, batch, torch.float16, dev) if use_ws else None
        run = lambda i: f(Wc[i % copies], M, K, x, out=y, flags=flags, workspace=wsp)
    else:
        x = synth.activations(batch, K, seed=2, dtype=torch.bfloat16, device=dev)
        f = gq.gq_gemm_q4_0 if fmt == "q4_0" else gq.gq_gemm_ksb
        y = torch.empty((batch, M), dtype=torch.float32, device=dev)
        run = lambda i: f(Wc[i % copies], M, K, x, out=y)
    for i in range(launches):
        run(i)
    torch.cuda.synchronize()
    print(json.dumps({"single": spec, "batch": batch, "launches": launches, "bytes": nb}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--copies", type=int, default=16)
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="bounded sample of oracle work for cpu_baseline")
    ap.add_argument("--suite", default=None,
                    help="also measure every hot-path row; JSON lines written to this file")
    ap.add_argument("--single", default=None,
                    help="profiling aid: launch one call a few times, e.g. gemv:q4_0:4096:11008, "
                         "grouped:q4_0:2, quantize:ksb:268435456")
    ap.add_argument("--launches", type=int, default=4)
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--flags", type=int, default=0)
    ap.add_argument("--workspace", action="store_true",
                    help="--single gemv: pass a workspace (the batch-1 integer path)")
    args = ap.parse_args()
    if args.single:
        run_single(args.single, args.launches, args.batch, args.flags, args.workspace)
        return

    rank, ws, local = dist_setup()
    try:
        if args.impl == "reference":
            res = run_reference(args, rank, ws)
        else:
            res = run_ours(args, rank, ws, local)
            if rank == 0 and ws == 1 and res is not None:
                v, cores, desc = OracleSample().run(args.cpu_seconds)
                res["cpu_baseline"] = {"value": round(v, 3), "unit": "GB/s", "cores": cores,
                                       "kind": "oracle", "sample": desc}
            if args.suite and rank == 0:
                run_suite(args.suite)
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
