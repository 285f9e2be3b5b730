#!/usr/bin/env python3
"""Benchmark of the batch-1 Q4 GEMV decode stream on B200.

Headline workload: batch-1 GEMV y = W_hat x over the 4096x11008 weight shape
in both Q4 formats and both orientations -- Q4_0 and super-block (ksb)
weights, M=4096 x K=11008 and M=11008 x K=4096 -- each over ``--copies``
distinct copies of its packed matrix, launched back to back (a CUDA graph of
``--chain`` launches cycling over the copies, programmatic dependent launch),
on both weight layouts the library serves:
canonical rows (gq_gemv_*) and tiled storage (gq_gemv_*_tiled, made once by
gq_repack_*).  A step is one pass over the four cases on both layouts; the
copies rotate over far more than the 126 MB L2, so every GEMV reads cold
weights.

Metric: streamed-weight GB/s = packed weight bytes / device time, per case.
``value`` is the worst of the four cases on the layout whose worst case is
higher; the other cases, the other layout and the remaining hot-path rows
(whole-model stream, batch 8, GEMM, quantize/dequantize, a plain read) are
further keys of the same JSON line, each with its fraction of the measured
peak.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (torchrun), every rank runs the same workload on its own GPU
(independent replicas: the path has no exchange step) and rank 0 prints the
aggregate over ranks with the max of the per-rank device times.
"""
from __future__ import annotations

import argparse
import hashlib
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
LAYOUTS = ("canonical", "tiled")
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0

# DRAM bytes (read + write) of one launch, from one ncu capture of that
# kernel on that case (bench.py --single, a cold launch).  Reported only while
# the kernel's sources hash to what was captured; a change to the kernel makes
# it null until it is captured again.
TRAFFIC = {
    "canonical ksb 4096 11008": {"bytes": 24349440, "sources": {
            "bit_gemv_q4_b200/csrc/gq_gemv.cu": "b6737f175c04b0f93c608fece7df7fed31a2b2d12f0bed7bba5339b9ec20c40e",
            "bit_gemv_q4_b200/csrc/gq_gemv.h": "91b29c15fbd80ae3ad2435b203453a1ba1d4da29da52322e6e996adb97cd8ebe",
            "bit_gemv_q4_b200/csrc/gq_device.cuh": "dc4d0fc96908a38ffd15ae87b6aecb7f02d029f2b003e9cbdae6614ee1f5e7a2"}},
    "tiled q4_0 4096 11008": {"bytes": 25420800, "sources": {
            "bit_gemv_q4_b200/csrc/gq_tiled.cu": "ef9b0561deae33b7305288cce25dfd501156aa1738d446a4e783e86696996c40",
            "bit_gemv_q4_b200/csrc/gq_device.cuh": "dc4d0fc96908a38ffd15ae87b6aecb7f02d029f2b003e9cbdae6614ee1f5e7a2",
            "bit_gemv_q4_b200/csrc/gq_tc.cuh": "b15f28de0672760637e15afae0059536e9c3acc85b1737d0e290acd10794f382"}},
    "tiled ksb 4096 11008": {"bytes": 24364032, "sources": {
            "bit_gemv_q4_b200/csrc/gq_tiled.cu": "ef9b0561deae33b7305288cce25dfd501156aa1738d446a4e783e86696996c40",
            "bit_gemv_q4_b200/csrc/gq_device.cuh": "dc4d0fc96908a38ffd15ae87b6aecb7f02d029f2b003e9cbdae6614ee1f5e7a2",
            "bit_gemv_q4_b200/csrc/gq_tc.cuh": "b15f28de0672760637e15afae0059536e9c3acc85b1737d0e290acd10794f382"}},
}


def traffic(layout, fmt, M, K):
    entry = TRAFFIC.get(f"{layout} {fmt} {M} {K}")
    if not entry:
        return None
    for rel, digest in entry["sources"].items():
        try:
            with open(os.path.join(ROOT, rel), "rb") as f:
                if hashlib.sha256(f.read()).hexdigest() != digest:
                    return None
        except OSError:
            return None
    return entry["bytes"]


def packed_bytes(fmt, M, K):
    return M * (K // 32 * 18 if fmt == "q4_0" else K // 256 * 138)


def measured_peaks():
    """(HBM GB/s, bf16 TFLOP/s burst, source)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


# ----------------------------------------------------------------- clocks
THROTTLE_BITS = {  # clock-event reason bit -> name (NVML and nvidia-smi agree)
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
    0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
    0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
    0x100: "display_clock_setting",
}


class ClockSampler:
    """SM clock and clock-event reasons of this process's GPU (found by UUID),
    read through NVML every `period` seconds while the run lasts; nvidia-smi
    at 10 ms if NVML is unavailable."""

    def __init__(self, device_index: int, period: float = 0.005):
        self.dev = device_index
        self.period = period
        self.samples = []  # (sm_mhz, sm_max_mhz, reason bits)
        self.stop = threading.Event()
        self.thread = None
        self.proc = None
        self.source = None

    def _uuid(self):
        import torch
        return "GPU-" + str(torch.cuda.get_device_properties(self.dev).uuid)

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByUUID(self._uuid())
            mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            reasons_fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons

            def loop():
                while not self.stop.is_set():
                    try:
                        sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                        bits = reasons_fn(h)
                        self.samples.append((float(sm), float(mx), int(bits)))
                    except Exception:
                        pass
                    self.stop.wait(self.period)

            self.thread = threading.Thread(target=loop, daemon=True)
            self.thread.start()
            self.source = f"NVML every {self.period * 1e3:.0f} ms"
        except Exception:
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", "--id=" + self._uuid(),
                     "--query-gpu=clocks.sm,clocks.max.sm,clocks_event_reasons.active",
                     "--format=csv,noheader,nounits", "-lms", "10"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                self.thread = threading.Thread(target=self._read_smi, daemon=True)
                self.thread.start()
                self.source = "nvidia-smi every 10 ms"
            except Exception:
                self.proc = None
        return self

    def _read_smi(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            try:
                self.samples.append((float(parts[0]), float(parts[1]), int(parts[2], 16)))
            except (ValueError, IndexError):
                continue

    def __exit__(self, *exc):
        self.stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self):
        busy = [s for s in self.samples if not (s[2] & 0x1)]
        use = busy or self.samples
        reasons = set()
        for _, _, bits in use:
            for b, name in THROTTLE_BITS.items():
                if bits & b and name != "gpu_idle":
                    reasons.add(name)
        if not use:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "source": self.source}
        return {"sm_mhz": statistics.median(s[0] for s in use),
                "sm_max_mhz": max(s[1] for s in use), "reasons": sorted(reasons),
                "samples": len(self.samples), "samples_busy": len(busy), "source": self.source}


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
def build_cases(gq, synth, copies, device):
    """Packed weight copies on both layouts, activations and outputs for the
    four headline cases."""
    import torch
    sets = []
    for ci, (fmt, M, K) in enumerate(CASES):
        code = gq.GQ_FMT_Q4_0 if fmt == "q4_0" else gq.GQ_FMT_KSB
        w = synth.gaussian_weights(M, K, seed=100 + ci, device=device)
        q = (gq.gq_quantize_q4_0 if fmt == "q4_0" else gq.gq_quantize_ksb)(w.view(-1))
        del w
        nb = packed_bytes(fmt, M, K)
        Wc = torch.empty((copies, nb), dtype=torch.uint8, device=device)
        Wc.copy_(q.view(1, nb).expand(copies, nb))
        Tc = torch.empty((copies, gq.gq_tiled_bytes(code, M, K)), dtype=torch.uint8, device=device)
        for c in range(copies):
            gq.gq_repack(code, Wc[c], M, K, out=Tc[c])
        x = synth.activations(1, K, seed=200 + ci, dtype=torch.float16, device=device)
        y = torch.empty((1, M), dtype=torch.float16, device=device)
        sets.append(dict(fmt=fmt, M=M, K=K, code=code, W=Wc, T=Tc, x=x, y=y, nbytes=nb,
                         canonical=gq.gq_gemv_q4_0 if fmt == "q4_0" else gq.gq_gemv_ksb,
                         tiled=gq.gq_gemv_q4_0_tiled if fmt == "q4_0" else gq.gq_gemv_ksb_tiled))
    torch.cuda.synchronize()
    return sets


def launch_case(s, layout, launches, flags):
    """`launches` GEMVs of one case through the C ABI, cycling over the
    weight copies."""
    mats = s["W"] if layout == "canonical" else s["T"]
    f = s[layout]
    for c in range(launches):
        f(mats[c % mats.shape[0]], s["M"], s["K"], s["x"], y_dtype=s["y"].dtype, out=s["y"],
          flags=flags)


def capture(fn):
    import torch
    fn()  # eager warm-up outside capture (sets kernel attributes)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


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


def _graph_ms(fn, reps):
    """Device ms per replay of a CUDA graph of fn()."""
    g = capture(fn)
    ms = _timed(g.replay, reps)
    del g
    return ms


def headline(args, sets, ws):
    """K steps; each case of each layout is one CUDA graph of `chain` PDL
    launches over the rotated copies, replayed K times in a row between two
    events.  Returns {(layout, case index): ms over the K replays (max over
    ranks)} and the whole region's ms."""
    import torch
    import bit_gemv_q4_b200 as gq
    chain, flags = args.chain, gq.GQ_GEMV_PDL
    graphs = {}
    for layout in LAYOUTS:
        for i, s in enumerate(sets):
            graphs[(layout, i)] = capture(lambda s=s, layout=layout: launch_case(s, layout, chain,
                                                                                flags))
    for g in graphs.values():
        for _ in range(args.warmup):
            g.replay()
    ev = {k: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for k in graphs}
    torch.cuda.synchronize()
    barrier(ws)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for k, g in graphs.items():
        ev[k][0].record()
        for _ in range(args.steps):
            g.replay()
        ev[k][1].record()
    t1.record()
    torch.cuda.synchronize()
    barrier(ws)
    ms = {k: max_over_ranks(e[0].elapsed_time(e[1]), ws) for k, e in ev.items()}
    total = max_over_ranks(t0.elapsed_time(t1), ws)
    del graphs
    return ms, total


def e2e_run(args, sets, layout, ws):
    """End to end through the public API with host buffers: every step copies
    the four activation vectors from pinned host memory, calls gq_gemv_* once
    per weight copy (eager, through the C ABI) and copies the four results
    back into pinned host memory.  Device time of the whole loop."""
    import torch
    import bit_gemv_q4_b200 as gq
    copies, flags = args.copies, gq.GQ_GEMV_PDL
    hx = [s["x"].cpu().pin_memory() for s in sets]
    hy = [torch.empty(s["y"].shape, dtype=s["y"].dtype).pin_memory() for s in sets]

    def step():
        for i, s in enumerate(sets):
            s["x"].copy_(hx[i], non_blocking=True)
        for s in sets:
            launch_case(s, layout, copies, flags)
        for i, s in enumerate(sets):
            hy[i].copy_(s["y"], non_blocking=True)

    steps = max(20, args.steps // 20)
    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    barrier(ws)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    barrier(ws)
    wbytes = sum(s["nbytes"] for s in sets) * copies
    gbs, _ = aggregate(wbytes * steps / 1e9, e0.elapsed_time(e1), ws)
    return {"value": round(gbs, 1), "unit": "GB/s",
            "h2d_bytes_per_step": sum(s["K"] * 2 for s in sets),
            "d2h_bytes_per_step": sum(s["M"] * 2 for s in sets),
            "mode": f"eager gq_gemv_*{'_tiled' if layout == 'tiled' else ''} calls, "
                    f"{len(sets) * copies} per step, pinned host copies in and out", "steps": steps}


def extra_rows(gq, synth, dev, peak, bf16):
    """The other hot-path rows, each on its own workload (CUDA events around
    CUDA graphs; weight copies rotated past the L2 where the row is a stream)."""
    import torch
    out = {}

    def quant(fmt, w):
        return (gq.gq_quantize_q4_0 if fmt == "q4_0" else gq.gq_quantize_ksb)(w.reshape(-1))

    def frac(gbs):
        return round(gbs / peak, 4)

    # whole-model weight stream: 32 layers x (4 x 4096^2 + 3 x 11008x4096), one x
    ms_rows = {}
    for fmt in ("q4_0", "ksb"):
        shapes = ([(4096, 4096)] * 4 + [(11008, 4096)] * 3) * 32
        mats, total = [], 0
        for i, (M, K) in enumerate(shapes):
            w = synth.gaussian_weights(M, K, seed=30000 + i, device=dev)
            mats.append((quant(fmt, w), M, K))
            total += mats[-1][0].numel()
            del w
        x = synth.activations(1, 4096, seed=9, dtype=torch.float16, device=dev)
        ys = {M: torch.empty((1, M), dtype=torch.float16, device=dev) for M in (4096, 11008)}
        f = gq.gq_gemv_q4_0 if fmt == "q4_0" else gq.gq_gemv_ksb
        ms = _graph_ms(lambda: [f(qm, M, K, x, out=ys[M], flags=gq.GQ_GEMV_PDL)
                                for qm, M, K in mats], 5)
        fg = gq.gq_gemv_q4_0_grouped if fmt == "q4_0" else gq.gq_gemv_ksb_grouped
        outs = [torch.empty((1, M), dtype=torch.float16, device=dev) for _, M, _ in mats]
        Ws, Ms = [m[0] for m in mats], [m[1] for m in mats]
        msg = _graph_ms(lambda: fg(Ws, Ms, 4096, x, outs=outs, flags=gq.GQ_GEMV_PDL), 5)
        # the same stream from tiled storage (each matrix repacked once)
        fmt_code = gq.GQ_FMT_Q4_0 if fmt == "q4_0" else gq.GQ_FMT_KSB
        Ts = [gq.gq_repack(fmt_code, qm, M, K) for qm, M, K in mats]
        ft = gq.gq_gemv_q4_0_tiled_grouped if fmt == "q4_0" else gq.gq_gemv_ksb_tiled_grouped
        mst = _graph_ms(lambda: ft(Ts, Ms, 4096, x, outs=outs, flags=gq.GQ_GEMV_PDL), 5)
        # one grouped call per decoder layer (its 7 matrices), 32 calls chained with PDL
        L = 7
        msl = _graph_ms(lambda: [fg(Ws[i:i + L], Ms[i:i + L], 4096, x, outs=outs[i:i + L],
                                    flags=gq.GQ_GEMV_PDL) for i in range(0, len(Ms), L)], 5)
        mstl = _graph_ms(lambda: [ft(Ts[i:i + L], Ms[i:i + L], 4096, x, outs=outs[i:i + L],
                                     flags=gq.GQ_GEMV_PDL) for i in range(0, len(Ms), L)], 5)
        g1, g2, g3 = (total / (t * 1e-3) / 1e9 for t in (ms, msg, mst))
        g4, g5 = (total / (t * 1e-3) / 1e9 for t in (msl, mstl))

        def row(t, g):
            return {"ms": round(t, 3), "gbs": round(g, 1), "frac_of_peak": frac(g),
                    "matrices_per_s": round(224 / (t * 1e-3), 1)}
        ms_rows[fmt] = {"weight_bytes": total, "graph": row(ms, g1), "grouped": row(msg, g2),
                        "grouped_tiled": row(mst, g3), "grouped_per_layer": row(msl, g4),
                        "grouped_tiled_per_layer": row(mstl, g5)}
        del mats, Ws, Ts, outs
        torch.cuda.empty_cache()
    out["model_stream"] = dict(
        workload="32 layers x (4 x 4096x4096 + 3 x 11008x4096) = 224 batch-1 GEMVs, x fp16; "
                 "'graph': one CUDA graph of 224 PDL launches, 'grouped': one grouped call, "
                 "'grouped_tiled': one grouped call on tiled storage; '*_per_layer': one "
                 "grouped call per layer (7 matrices), 32 calls chained with PDL in one graph "
                 "(weight_bytes: the canonical bytes, the same for both layouts)",
        **ms_rows)

    # batch 8 on the MLP shape, and the tensor-core GEMM on the same W
    M, K = 11008, 4096
    b8, gemm = {}, {}
    for fmt in ("q4_0", "ksb"):
        w = synth.gaussian_weights(M, K, seed=11, device=dev) if fmt == "q4_0" else \
            synth.logstd_weights(M, K, seed=2, device=dev)
        q = quant(fmt, w)
        del w
        nb = q.numel()
        copies = 6
        Wc = torch.empty((copies, nb), dtype=torch.uint8, device=dev)
        Wc.copy_(q.view(1, nb).expand(copies, nb))
        x8 = synth.activations(8, K, seed=8, dtype=torch.float16, device=dev)
        y8 = torch.empty((8, M), dtype=torch.float16, device=dev)
        f = gq.gq_gemv_q4_0 if fmt == "q4_0" else gq.gq_gemv_ksb
        ms = _graph_ms(lambda: [f(Wc[i], M, K, x8, out=y8, flags=gq.GQ_GEMV_PDL)
                                for i in range(copies)], 20) / copies
        gbs = nb / (ms * 1e-3) / 1e9
        b8[fmt] = {"us": round(ms * 1e3, 3), "gbs": round(gbs, 1), "frac_of_peak": frac(gbs),
                   "tflops": round(2 * M * K * 8 / (ms * 1e-3) / 1e12, 3)}
        fm = gq.gq_gemm_q4_0 if fmt == "q4_0" else gq.gq_gemm_ksb
        gemm[fmt] = {}
        for B in (16, 64, 256):
            X = synth.activations(B, K, seed=12, dtype=torch.bfloat16, device=dev)
            Y = torch.empty((B, M), dtype=torch.float32, device=dev)
            wsp = torch.zeros(max(gq.gq_gemm_workspace_bytes(
                gq.GQ_FMT_Q4_0 if fmt == "q4_0" else gq.GQ_FMT_KSB, M, K, B), 1),
                dtype=torch.uint8, device=dev)
            ms = _graph_ms(lambda: [fm(Wc[i], M, K, X, out=Y, workspace=wsp)
                                    for i in range(copies)], 10) / copies
            tf = 2.0 * M * K * B / (ms * 1e-3) / 1e12
            gemm[fmt][str(B)] = {"us": round(ms * 1e3, 2), "tflops": round(tf, 1),
                                 "frac_of_bf16_peak": round(tf / bf16, 4),
                                 "weight_gbs": round(nb / (ms * 1e-3) / 1e9, 1)}
        del Wc
    out["batch8"] = dict(workload="W 11008x4096, X fp16 [8, 4096], Y fp16, 6 rotated copies", **b8)

    # small batches on the transposed shape, where x of 6..16 rows no longer
    # fits beside the weight ring: K split over clusters of 2..3 CTAs
    M, K = 4096, 11008
    bk = {}
    for fmt in ("q4_0", "ksb"):
        w = synth.gaussian_weights(M, K, seed=13, device=dev) if fmt == "q4_0" else \
            synth.logstd_weights(M, K, seed=3, device=dev)
        q = quant(fmt, w)
        del w
        nb = q.numel()
        copies = 6
        Wc = torch.empty((copies, nb), dtype=torch.uint8, device=dev)
        Wc.copy_(q.view(1, nb).expand(copies, nb))
        f = gq.gq_gemv_q4_0 if fmt == "q4_0" else gq.gq_gemv_ksb
        fm = gq.gq_gemm_q4_0 if fmt == "q4_0" else gq.gq_gemm_ksb
        bk[fmt] = {}
        for B in (2, 4, 8, 16):
            if B <= 8:
                xb = synth.activations(B, K, seed=B, dtype=torch.float16, device=dev)
                yb = torch.empty((B, M), dtype=torch.float16, device=dev)
                ms = _graph_ms(lambda: [f(Wc[i], M, K, xb, out=yb, flags=gq.GQ_GEMV_PDL)
                                        for i in range(copies)], 20) / copies
            else:
                xb = synth.activations(B, K, seed=B, dtype=torch.bfloat16, device=dev)
                yb = torch.empty((B, M), dtype=torch.float32, device=dev)
                wsp = torch.zeros(max(gq.gq_gemm_workspace_bytes(
                    gq.GQ_FMT_Q4_0 if fmt == "q4_0" else gq.GQ_FMT_KSB, M, K, B), 1),
                    dtype=torch.uint8, device=dev)
                ms = _graph_ms(lambda: [fm(Wc[i], M, K, xb, out=yb, workspace=wsp)
                                        for i in range(copies)], 20) / copies
            gbs = nb / (ms * 1e-3) / 1e9
            bk[fmt][str(B)] = {"us": round(ms * 1e3, 3), "gbs": round(gbs, 1),
                               "frac_of_peak": frac(gbs)}
        del Wc
    out["batches_4096x11008"] = dict(
        workload="W 4096x11008, X [B, 11008] (fp16 through gq_gemv_* for B <= 8 with PDL, bf16 "
                 "through gq_gemm_* for B = 16), 6 rotated copies", **bk)
    out["gemm"] = dict(workload="W 11008x4096, X bf16 [B, 4096], Y fp32, 6 rotated copies; "
                                "useful flops 2*M*K*B", **gemm)

    # quantize and dequantize 1e9 weights ~ N(0, 0.02^2)
    n = 1_000_000_000
    w = synth.gaussian_weights(n // 8000, 8000, seed=4, frac=0.0, device=dev).view(-1)
    qd = {}
    for fmt, nbytes in (("q4_0", n // 32 * 18), ("ksb", n // 256 * 138)):
        q = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        fq = gq.gq_quantize_q4_0 if fmt == "q4_0" else gq.gq_quantize_ksb
        fd = gq.gq_dequantize_q4_0 if fmt == "q4_0" else gq.gq_dequantize_ksb
        row = {}
        for kind, fn in (("quantize", lambda: fq(w, out=q)), ("dequantize", lambda: fd(q, n, out=w))):
            ms = _timed(fn, 5)
            gbs = (4 * n + nbytes) / (ms * 1e-3) / 1e9
            row[kind] = {"ms": round(ms, 3), "tbs": round(gbs / 1e3, 3), "frac_of_peak": frac(gbs),
                         "gweights_per_s": round(n / (ms * 1e-3) / 1e9, 2)}
        qd[fmt] = row
        del q
    del w
    torch.cuda.empty_cache()
    out["quantize_dequantize"] = dict(workload="1e9 fp32 weights <-> packed bytes; bytes = 4n + "
                                               "packed", **qd)
    return out


def plain_read(args, sets, peak):
    """The same weight copies read once each by a plain streaming-read
    kernel (gq_stream_read), one launch per matrix, no PDL, same graph
    method: a reference point for the GEMV launches, not a ceiling for them
    (the GEMV chain uses PDL)."""
    import torch
    import bit_gemv_q4_b200 as gq
    dev = sets[0]["W"].device
    sink = torch.zeros(1, dtype=torch.int32, device=dev)
    res = {}
    for s in sets:
        ms = _graph_ms(lambda s=s: [gq.gq_stream_read(s["W"][c], sink) for c in range(args.copies)],
                       max(10, args.steps // 50)) / args.copies
        gbs = s["nbytes"] / (ms * 1e-3) / 1e9
        res[f"{s['fmt']} M={s['M']} K={s['K']}"] = {"gbs": round(gbs, 1),
                                                     "frac_of_peak": round(gbs / peak, 4)}
    return res


def run_ours(args, rank, ws, local):
    import torch
    import bit_gemv_q4_b200 as gq
    import synth

    dev = torch.device("cuda", torch.cuda.current_device())
    peak, bf16, peak_src = measured_peaks()
    copies = args.copies
    with ClockSampler(local) as clk:
        sets = build_cases(gq, synth, copies, dev)
        ms, total_ms = headline(args, sets, ws)

        per = {}
        for layout in LAYOUTS:
            per[layout] = {}
            for i, s in enumerate(sets):
                gemv_us = ms[(layout, i)] * 1e3 / (args.steps * args.chain)
                gbs = s["nbytes"] / (gemv_us * 1e-6) / 1e9
                per[layout][i] = (gbs, gemv_us)
        worst = {lay: min(range(len(sets)), key=lambda i: per[lay][i][0]) for lay in LAYOUTS}
        lead = max(LAYOUTS, key=lambda lay: per[lay][worst[lay]][0])
        wi = worst[lead]
        ws_case = sets[wi]
        value = per[lead][wi][0] * ws  # whole job: every rank streams the same bytes
        # the dominant kernel: the headline layout's kernel on the worst case
        algo_launch = ws_case["nbytes"] + ws_case["K"] * 2 + ws_case["M"] * 2
        achieved = algo_launch / (per[lead][wi][1] * 1e-6) / 1e9

        e2e = e2e_run(args, sets, lead, ws)
        extras = extra_rows(gq, synth, dev, peak, bf16) if (rank == 0 and not args.no_extras) else {}
        reads = plain_read(args, sets, peak) if rank == 0 else {}
    barrier(ws)

    def case_table(layout):
        return {f"{s['fmt']} M={s['M']} K={s['K']}": {
            "gbs": round(per[layout][i][0], 1), "us_per_gemv": round(per[layout][i][1], 3),
            "frac_of_peak": round(per[layout][i][0] / peak, 4)} for i, s in enumerate(sets)}

    all_bytes = sum(s["nbytes"] for s in sets) * args.chain
    lead_ms = sum(ms[(lead, i)] for i in range(len(sets)))
    kernel = {"canonical": "gemv_kernel (gq_gemv_q4_0 / gq_gemv_ksb)",
              "tiled": "gemv_tiled_kernel (gq_gemv_q4_0_tiled / gq_gemv_ksb_tiled)"}
    result = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f16", "data": "synthetic",
        "config": {
            "workload": ("batch-1 GEMV, Q4_0 and super-block weights, 4096x11008 in both "
                         "orientations (M=4096 K=11008 and M=11008 K=4096), x fp16, y fp16, "
                         f"{copies} copies of each matrix; value = the worst of the four cases"),
            "headline_case": f"{ws_case['fmt']} M={ws_case['M']} K={ws_case['K']}",
            "headline_layout": lead,
            "step": "one pass over the four cases on both layouts (canonical rows and tiled "
                    f"storage), {2 * len(sets) * args.chain} GEMVs",
            "chain": f"{args.chain} GEMVs per CUDA graph, cycling over the {copies} copies",
            "l2": "inputs larger than L2 (each case rotates over %.2f GB of copies)"
                  % (min(s["nbytes"] for s in sets) * copies / 1e9),
            "launch": "CUDA graph per case and layout, programmatic dependent launch",
            "parallelism": "replicas" if ws > 1 else "single GPU",
        },
        "frac_of_peak": round(value / ws / peak, 4),
        "frac_of_nominal_8tbs": round(value / ws / 8000.0, 4),
        "all_cases_gbs": round(all_bytes * args.steps / (lead_ms * 1e-3) / 1e9 * ws, 1),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                     "peak_source": f"{peak_src} hbm_gbs (burst copy)", "unit": "GB/s",
                     "frac": round(achieved / peak, 4),
                     "traffic": traffic(lead, ws_case["fmt"], ws_case["M"], ws_case["K"]),
                     "kernel": kernel[lead] + f" on {ws_case['fmt']} M={ws_case['M']} "
                                              f"K={ws_case['K']}",
                     "algorithmic_bytes_per_launch": algo_launch},
        "cases": {layout: case_table(layout) for layout in LAYOUTS},
        "e2e": e2e,
        "gpu_launches": 2 * len(sets) * args.chain * args.steps,
        "clocks": clk.summary(),
    }
    if extras:
        result.update(extras)
    if reads:
        result["plain_read"] = dict(
            what="the same weight copies, one plain streaming-read launch (gq_stream_read) per "
                 "matrix, no PDL: a reference point for the GEMV launches, not a ceiling", **reads)
    return result


# ---------------------------------------------------- the oracle on the host
def all_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


class OracleSample:
    """The four headline cases (one matrix each), quantized by the oracle;
    ``run`` times the oracle's product over them on the host cores."""

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

    def run(self, seconds: float, threads: int | None = None):
        """Whole passes over the four cases until `seconds` have passed;
        returns (GB/s of packed weights, threads, description)."""
        threads = threads or all_cores()
        self.oracle.set_threads(threads)
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
                f"one matrix each) in {el:.1f} s on {threads} thread(s)")
        return nbytes / el / 1e9, threads, desc


def _best(fn, reps):
    best = None
    for _ in range(reps):
        t0 = time.perf_counter()
        fn()
        el = time.perf_counter() - t0
        best = el if best is None else min(best, el)
    return best


def oracle_configs():
    """The oracle timed on each configuration's workload: 1 core and all
    cores for the single-matrix configurations, all cores for the model
    stream, the GEMM and quantize (bounded samples, scaled to the metric's
    unit and named).  steady clock (perf_counter), best of 3 where small."""
    import numpy as np
    import oracle
    import synth
    import torch
    oracle.build()
    n_all = all_cores()
    out = {"cores_available": n_all}

    def both(fn, units, unit, reps=3):
        r = {}
        for th in (1, n_all):
            oracle.set_threads(th)
            el = _best(fn, reps)
            r[f"{th}_core{'s' if th > 1 else ''}"] = round(units / el, 4)
        return dict(unit=unit, **r)

    # config 1: W fp32 256x1024 -> Q4_0, x fp32, y fp32
    w = synth.gaussian_weights(256, 1024, seed=0).numpy().ravel()
    q, _ = oracle.quantize(oracle.FMT_Q4_0, w)
    x = np.random.default_rng(0).standard_normal(1024).astype(np.float32)
    out["cfg1_gemv_256x1024"] = both(lambda: oracle.gemm(oracle.FMT_Q4_0, q, 256, 1024, x),
                                     q.size / 1e9, "GB/s")
    # config 2: 4096x4096 Q4_0, x fp16
    w = synth.gaussian_weights(4096, 4096, seed=1).numpy().ravel()
    q, _ = oracle.quantize(oracle.FMT_Q4_0, w)
    x = synth.activations(1, 4096, seed=1, dtype=torch.float16).numpy()
    out["cfg2_gemv_4096x4096_q4_0"] = both(lambda: oracle.gemm(oracle.FMT_Q4_0, q, 4096, 4096, x),
                                           q.size / 1e9, "GB/s")
    # config 3: 11008x4096 ksb, B = 1 and 8
    w = synth.logstd_weights(11008, 4096, seed=2).numpy().ravel()
    q, _ = oracle.quantize(oracle.FMT_KSB, w)
    for B in (1, 8):
        x = synth.activations(B, 4096, seed=3, dtype=torch.float16).numpy()
        out[f"cfg3_gemv_11008x4096_ksb_B{B}"] = both(
            lambda x=x, B=B: oracle.gemm(oracle.FMT_KSB, q, 11008, 4096, x), q.size / 1e9, "GB/s",
            reps=1 if B > 1 else 3)
    oracle.set_threads(n_all)
    # config 4: the model stream, sampled as one matrix of each shape per format,
    # weighted as a decoder layer (4 x 4096x4096 + 3 x 11008x4096)
    for fmt, f in (("q4_0", oracle.FMT_Q4_0), ("ksb", oracle.FMT_KSB)):
        x = synth.activations(1, 4096, seed=9, dtype=torch.float16).numpy()
        t_layer, nb_layer = 0.0, 0
        for i, (M, count) in enumerate(((4096, 4), (11008, 3))):
            w = synth.gaussian_weights(M, 4096, seed=30000 + 4 * i).numpy().ravel()
            qm = oracle.quantize(f, w)[0]
            t_layer += count * _best(lambda: oracle.gemm(f, qm, M, 4096, x), 1)
            nb_layer += count * qm.size
        out[f"cfg4_model_stream_{fmt}"] = {
            "unit": "GB/s", f"{n_all}_cores": round(nb_layer / t_layer / 1e9, 4),
            "matrices_per_s": round(7 / t_layer, 2),
            "sample": "one 4096x4096 and one 11008x4096 matrix, weighted 4:3 as in a layer"}
    # config 5: GEMM on sampled rows; quantize 1e8 of the 1e9 weights
    w = synth.gaussian_weights(11008, 4096, seed=11).numpy().ravel()
    q, _ = oracle.quantize(oracle.FMT_Q4_0, w)
    rows = np.arange(0, 11008, 11008 // 512, dtype=np.int64)[:512]
    for B in (16, 64, 256):
        X = synth.activations(B, 4096, seed=12, dtype=torch.bfloat16)
        xo = X.view(torch.int16).numpy().view(np.uint16)
        el = _best(lambda: oracle.gemm_rows(oracle.FMT_Q4_0, q, 11008, 4096, xo, rows,
                                            oracle.BF16), 1)
        out[f"cfg5_gemm_B{B}_q4_0"] = {"unit": "GFLOP/s",
                                       f"{n_all}_cores": round(2 * rows.size * 4096 * B / el / 1e9, 3),
                                       "sample": f"{rows.size} of the 11008 rows"}
    n = 100_000_000
    w = synth.gaussian_weights(n // 8000, 8000, seed=4, frac=0.0).numpy().ravel()
    for fmt, f, per in (("q4_0", oracle.FMT_Q4_0, 18 / 32), ("ksb", oracle.FMT_KSB, 138 / 256)):
        el = _best(lambda f=f: oracle.quantize(f, w), 1)
        out[f"cfg5_quantize_{fmt}"] = {"unit": "GB/s",
                                       f"{n_all}_cores": round(n * (4 + per) / el / 1e9, 3),
                                       "sample": "1e8 of the 1e9 weights"}
    return out


def run_reference(args, rank, ws):
    """The oracle as it stands, on this host's cores, same metric and config;
    each step is one pass over the four cases."""
    if rank != 0:
        return None
    smp = OracleSample()
    for _ in range(args.warmup):
        smp.run(0.0)
    vals, t0 = [], time.perf_counter()
    cores = all_cores()
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


def run_single(spec, launches, batch, flags, use_ws=False):
    """A few launches of one hot-path call (for profilers).  spec:
    "gemv:q4_0:4096:11008" / "tgemv:ksb:4096:11008" (canonical rows / tiled
    storage) / "gemm:ksb:11008:4096" (distinct copies of one matrix),
    "grouped:q4_0:<layers>" (the decoder-layer matrices 4 x 4096x4096 +
    3 x 11008x4096 per layer in one grouped call), or "quantize:ksb:<n>" /
    "dequantize:q4_0:<n>" (n weights)."""
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
    code = gq.GQ_FMT_Q4_0 if fmt == "q4_0" else gq.GQ_FMT_KSB
    w = synth.gaussian_weights(M, K, seed=1, device=dev)
    q = (gq.gq_quantize_q4_0 if fmt == "q4_0" else gq.gq_quantize_ksb)(w.view(-1))
    del w
    nb = q.numel()
    copies = 6
    Wc = torch.empty((copies, nb), dtype=torch.uint8, device=dev)
    Wc.copy_(q.view(1, nb).expand(copies, nb))
    if kind in ("gemv", "tgemv"):
        x = synth.activations(batch, K, seed=2, dtype=torch.float16, device=dev)
        y = torch.empty((batch, M), dtype=torch.float16, device=dev)
        if kind == "tgemv":
            Tc = torch.empty((copies, gq.gq_tiled_bytes(code, M, K)), dtype=torch.uint8, device=dev)
            for c in range(copies):
                gq.gq_repack(code, Wc[c], M, K, out=Tc[c])
            del Wc
            f = gq.gq_gemv_q4_0_tiled if fmt == "q4_0" else gq.gq_gemv_ksb_tiled
            run = lambda i: f(Tc[i % copies], M, K, x, out=y, flags=flags)
        else:
            f = gq.gq_gemv_q4_0 if fmt == "q4_0" else gq.gq_gemv_ksb
            wsp = None
            if use_ws:
                need = gq.gq_gemv_workspace_bytes(code, M, K, batch, torch.float16)
                wsp = torch.zeros(need, dtype=torch.uint8, device=dev) if need else None
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
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--copies", type=int, default=16)
    ap.add_argument("--chain", type=int, default=64,
                    help="GEMVs per CUDA graph of a case (cycling over the copies)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="bounded sample of oracle work for cpu_baseline")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the non-headline rows and the per-configuration oracle timings")
    ap.add_argument("--single", default=None,
                    help="profiling aid: launch one call a few times, e.g. gemv:q4_0:4096:11008, "
                         "tgemv:q4_0:4096:11008, grouped:q4_0:2, quantize:ksb:268435456")
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
                if not args.no_extras:
                    res["cpu_baselines"] = oracle_configs()
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
