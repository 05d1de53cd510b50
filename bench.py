#!/usr/bin/env python
"""Benchmark of the ternary weight-only grouped linear layer on B200.

Headline (`value`): decode GEMV throughput in GB/s of algorithmic HBM bytes
(packed codes + fp16 scales + bf16 activations + bf16 outputs) on the
Qwen3.5-0.8B-shaped FFN projections (gate/up 3584 x 1024, down 1024 x 3584),
G in {64, 128}, M = 1.  One step = a decode token through a 48-layer stack of
those three projections for both group sizes (288 tq_gemv launches replayed
from one CUDA graph).  The stack's working set (232 MB) exceeds the 126 MB L2,
so no step finds its weights in cache.

The other rows of the hot path are measured in the same run and reported in
their own keys: bulk quantize+pack and unpack over the 72-matrix, 24-layer FFN
stack (packed-byte GB/s both ways), a single large streaming GEMV, and the
tensor-core prefill GEMM (M=4096, 4096->14336 and 14336->4096, TFLOP/s).

Multi-GPU: one process per GPU (torchrun), every rank runs its own replica
(weak scaling, no data-path collective); time = max over ranks.
`--impl reference` times the CPU oracle on a bounded sample of the same
workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "ternary x bf16 GEMV HBM GB/s (% of peak); prefill GEMM TFLOP/s; pack GB/s"
# DRAM bytes (read + write) of one gemv_predecode_kernel launch per decode
# shape (N, K, G), M=1, from an ncu capture of dram__bytes_read.sum +
# dram__bytes_write.sum on `bench.py --only traffic` (one launch per shape,
# caches flushed by ncu before each; the bf16 Y stays in L2, 0 bytes written).
# Valid only for the kernel source they were captured on: the SHA-256 of
# gemv_predecode.cu at capture time is recorded beside them, and the figures
# are reported only while the current source still has that hash.
PREDECODE_DRAM_BYTES = {(3584, 1024, 64): 902912, (1024, 3584, 64): 907008,
                        (3584, 1024, 128): 845312, (1024, 3584, 128): 850176}
PREDECODE_DRAM_SRC_SHA256 = "23cc404f71359f660e2b572e039476d724c2f30550d7fb53e89881631436f091"
FFN = {"gate": (3584, 1024), "up": (3584, 1024), "down": (1024, 3584)}
MSWEEP = {"q": (1536, 1536), "o": (1536, 1536), "gate": (4096, 1536), "up": (4096, 1536), "down": (1536, 4096)}
MSWEEP_LAYERS = 28
MSWEEP_M = (1, 2, 4, 8, 16, 32, 64)
GROUPS = (64, 128)
LAYERS = 48
L2_BYTES = 126 * 1024 * 1024


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def source_sha256(rel):
    import hashlib
    with open(os.path.join(ROOT, rel), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


def traffic_valid() -> bool:
    """True while gemv_predecode.cu is the source the recorded DRAM bytes were captured on."""
    return (PREDECODE_DRAM_SRC_SHA256 is not None and
            source_sha256("ternary_weight_only_group_b200/csrc/gemv_predecode.cu") == PREDECODE_DRAM_SRC_SHA256)


def host_cpu():
    """Model name, logical CPUs and the CPUs this process may run on."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        affinity = len(os.sched_getaffinity(0))
    except AttributeError:
        affinity = os.cpu_count()
    return {"model": model, "logical_cpus": os.cpu_count(), "affinity_cpus": affinity}


def packed_bytes(N, K, G):
    return N * (K // G) * ((G + 4) // 5) + N * (K // G) * 2


def packed2_bytes(N, K, G):
    """Codes + scales of the 2-bit format (four codes per byte)."""
    return N * (K // G) * ((G + 3) // 4) + N * (K // G) * 2


# --------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=2)

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            parts = [p.strip() for p in l.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------- helpers

def dist_setup(args):
    import torch
    import torch.distributed as dist
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and not dist.is_initialized():
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=60))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def timed(fn, steps, warmup, world, stream=None):
    """W untimed + K timed calls of fn, barrier + synchronize on both sides,
    CUDA events on the launching stream; returns max-over-ranks ms."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    s = stream or torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push("timed")
    e0.record(s)
    for _ in range(steps):
        fn()
    e1.record(s)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    barrier(world)
    ms = e0.elapsed_time(e1)
    return max_over_ranks(ms, world)


def timed_flushed(fn, steps, warmup, world):
    """Like timed(), for a kernel whose inputs fit in L2: before every call a
    256 MB buffer is written (evicting L2), and only the call itself sits
    between its pair of CUDA events; returns the max-over-ranks sum in ms."""
    import torch
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    for _ in range(warmup):
        flush.zero_()
        fn()
    torch.cuda.synchronize()
    barrier(world)
    s = torch.cuda.current_stream()
    pairs = []
    torch.cuda.nvtx.range_push("timed")
    for _ in range(steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        fn()
        e1.record(s)
        pairs.append((e0, e1))
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    barrier(world)
    ms = sum(a.elapsed_time(b) for a, b in pairs)
    del flush
    return max_over_ranks(ms, world)


def device_weights(N, K, seed, outliers=True):
    """Seeded synthetic bf16 weights ~ N(0, 0.02), 0.1% of entries x10, made on the device."""
    import torch
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    w = torch.randn((N, K), generator=g, device="cuda", dtype=torch.float32) * 0.02
    if outliers:
        mask = torch.rand((N, K), generator=g, device="cuda") < 1e-3
        w = torch.where(mask, w * 10.0, w)
    return w.to(torch.bfloat16)


def device_acts(M, K, seed):
    import torch
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    return torch.randn((M, K), generator=g, device="cuda", dtype=torch.float32).to(torch.bfloat16)


# --------------------------------------------------------------------- our arm

def build_decode_stack(tq, layers, pack="base3"):
    """Packed weights of `layers` x (gate, up, down) for each G, plus one X
    buffer and one Y buffer sliced per launch (so a whole step's inputs and
    outputs are single contiguous transfers for the end-to-end measurement)."""
    import torch
    calls = []
    x_elems = y_elems = 0
    for G in GROUPS:
        for l in range(layers):
            for name, (N, K) in FFN.items():
                calls.append((G, l, name, N, K, x_elems, y_elems))
                x_elems += K
                y_elems += N
    packs = {}
    for G in GROUPS if pack else ():
        for l in range(layers):
            for i, (name, (N, K)) in enumerate(FFN.items()):
                W = device_weights(N, K, seed=1000 + 3 * l + i)
                packs[(G, l, name)] = tq.quantize_pack(W, G)
                del W
    X = device_acts(1, x_elems, seed=2001).view(-1)
    Y = torch.empty(y_elems, dtype=torch.bfloat16, device="cuda")
    torch.cuda.synchronize()
    return calls, packs, X, Y


def run_ours(args, rank, world, local):
    import torch
    import ternary_weight_only_group_b200 as tq
    from ternary_weight_only_group_b200 import _build
    if not _build.up_to_date():
        raise RuntimeError("libtq.so is missing or stale; run __graft_entry__.build() first")
    torch.cuda.set_device(local)
    peaks = load_peaks()
    K_steps, W_steps = args.steps, args.warmup

    calls, packs, X, Y = build_decode_stack(tq, LAYERS)
    step_bytes = 0
    for (G, l, name, N, K, xo, yo) in calls:
        step_bytes += packed_bytes(N, K, G) + 2 * K + 2 * N

    def step_kernels():
        for (G, l, name, N, K, xo, yo) in calls:
            codes, scales = packs[(G, l, name)]
            tq.gemv(X[xo:xo + K].view(1, K), codes, scales, N, K, G,
                    out=Y[yo:yo + N].view(1, N))

    # warm once outside capture (sets kernel attributes), then capture one step
    step_kernels()
    torch.cuda.synchronize()
    cap = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=cap, capture_error_mode="relaxed"):
        step_kernels()
    torch.cuda.synchronize()

    # end-to-end variant: pinned host X in, kernels, pinned host Y out
    X_host = torch.empty(X.numel(), dtype=torch.bfloat16, pin_memory=True)
    X_host.copy_(X.cpu())
    Y_host = torch.empty(Y.numel(), dtype=torch.bfloat16, pin_memory=True)
    graph_e2e = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_e2e, stream=cap, capture_error_mode="relaxed"):
        X.copy_(X_host, non_blocking=True)
        step_kernels()
        Y_host.copy_(Y, non_blocking=True)
    torch.cuda.synchronize()

    launches_per_step = len(calls)
    results = {}
    with ClockSampler(local) as clocks:
        ms = timed(graph.replay, K_steps, W_steps, world)
        ms_e2e = timed(graph_e2e.replay, K_steps, W_steps, world)
        results["fused_gateup"] = bench_fused_gateup(tq, args, world, peaks, packs)
        results["stream"] = bench_gemv_stream(tq, args, world, peaks)
        results["pack"], results["unpack"] = bench_bulk_codec(tq, args, world, peaks)
        results["prefill"] = bench_prefill(tq, args, world, peaks)
        results["msweep"] = bench_msweep(tq, args, world, peaks)
        results["small_m_stack"] = bench_small_m_stack(tq, args, world, peaks)
        results["ternary2"] = bench_ternary2(tq, args, world, peaks)
        results["w4"] = bench_w4(tq, args, world, peaks)
    clk = clocks.summary()

    ms_step = ms / K_steps
    value = world * step_bytes * K_steps / (ms * 1e-3) / 1e9
    e2e = world * step_bytes * K_steps / (ms_e2e * 1e-3) / 1e9
    per_launch_us = ms_step * 1e3 / launches_per_step
    avg_bytes = step_bytes / launches_per_step
    traffic = None  # measured DRAM bytes per launch, averaged like avg_bytes
    if traffic_valid() and all((N, K, G) in PREDECODE_DRAM_BYTES for (G, l, name, N, K, xo, yo) in calls):
        traffic = round(sum(PREDECODE_DRAM_BYTES[(N, K, G)] for (G, l, name, N, K, xo, yo) in calls) / len(calls), 1)
    achieved = avg_bytes / (per_launch_us * 1e-6) / 1e9
    if rank != 0:
        return
    cpu = cpu_baseline(args)
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": K_steps,
        "warmup": W_steps,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic",
        "config": {
            "workload": "decode GEMV, M=1, Qwen3.5-0.8B-shaped FFN gate/up 3584x1024 and "
                        "down 1024x3584, G in {64,128}; one step = 48 layers x 3 projections "
                        "x 2 group sizes = 288 tq_gemv launches from one CUDA graph",
            "layers": LAYERS, "group_sizes": list(GROUPS), "M": 1, "out_dtype": "bf16",
            "l2": f"inputs larger than L2: {step_bytes / 1e6:.1f} MB per step vs 126 MB L2",
            "parallelism": f"replicas x{world}",
        },
        "roofline": {
            "bound": "hbm", "kernel": "gemv_predecode_kernel (tq_gemv, M=1)",
            "achieved": round(achieved, 2), "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": round(achieved / peaks["hbm_gbs"], 4),
            "peak_source": peaks["source"],
            "per_launch_us": round(per_launch_us, 3),
            "bytes_per_launch": round(avg_bytes, 1),
            "traffic": traffic,
        },
        "cpu_baseline": cpu,
        "e2e": {"value": round(e2e, 2), "unit": "GB/s",
                "h2d_bytes_per_step": X.numel() * 2, "d2h_bytes_per_step": Y.numel() * 2},
        "gpu_launches": launches_per_step * K_steps * 2 + count_launches(results),
        "clocks": clk,
        "fused_gateup": results["fused_gateup"],
        "gemv_stream": results["stream"],
        "pack": results["pack"],
        "unpack": results["unpack"],
        "prefill_gemm": results["prefill"],
        "msweep": results["msweep"],
        "small_m_stack": results["small_m_stack"],
        "ternary2": results["ternary2"],
        "w4": results["w4"],
    }
    print(json.dumps(line), flush=True)


def bench_fused_gateup(tq, args, world, peaks, packs):
    """The headline's decode chain with gate and up of every layer stacked
    into one [7168 x 1024] matrix (one launch sharing the activations) and
    down after it: 48 layers x 2 launches x 2 group sizes = 192 tq_gemv
    launches per step from one CUDA graph, the same weights and bytes."""
    import torch
    calls = []
    x_elems = y_elems = 0
    fused = {}
    for G in GROUPS:
        for l in range(LAYERS):
            cg_, sg = packs[(G, l, "gate")]
            cu, su = packs[(G, l, "up")]
            fused[(G, l)] = (torch.cat([cg_, cu]), torch.cat([sg, su]))
            for name, (N, K) in (("gateup", (2 * FFN["gate"][0], FFN["gate"][1])), ("down", FFN["down"])):
                calls.append((G, l, name, N, K, x_elems, y_elems))
                x_elems += K
                y_elems += N
    X = device_acts(1, x_elems, seed=2002).view(-1)
    Y = torch.empty(y_elems, dtype=torch.bfloat16, device="cuda")
    step_bytes = sum(packed_bytes(N, K, G) + 2 * K + 2 * N for (G, l, name, N, K, xo, yo) in calls)

    def step():
        for (G, l, name, N, K, xo, yo) in calls:
            c, s_ = fused[(G, l)] if name == "gateup" else packs[(G, l, "down")]
            tq.gemv(X[xo:xo + K].view(1, K), c, s_, N, K, G, out=Y[yo:yo + N].view(1, N))
    step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, capture_error_mode="relaxed"):
        step()
    ms = timed(graph.replay, args.steps, args.warmup, world)
    us = ms * 1e3 / args.steps
    gbs = step_bytes / us / 1e3
    del graph, fused
    return {"launches_per_step": len(calls), "us_per_step": round(us, 1),
            "us_per_launch": round(us / len(calls), 3), "GB/s": round(gbs, 1),
            "frac": round(gbs / peaks["hbm_gbs"], 4), "bytes_per_step": step_bytes,
            "launches": args.steps * len(calls),
            "note": "gate and up of each layer as one [7168 x 1024] launch, then down; both G"}


def count_launches(obj) -> int:
    """Sum of every "launches" entry in a (nested) result dict."""
    if isinstance(obj, dict):
        return sum(v if k == "launches" and isinstance(v, int) else count_launches(v) for k, v in obj.items())
    return 0


def graph_launch_us(launches, rounds, args, world):
    """Capture `rounds` passes over `launches` (one kernel launch each) in one
    CUDA graph and time its replays: microseconds per launch with launches
    back to back (programmatic dependency edges between them), not limited
    by the Python dispatcher."""
    import torch
    for f in launches:
        f()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, capture_error_mode="relaxed"):
        for _ in range(rounds):
            for f in launches:
                f()
    steps = max(3, args.steps)
    ms = timed(graph.replay, steps, max(3, args.warmup), world)
    del graph
    return ms * 1e3 / (steps * rounds * len(launches))


def bench_gemv_stream(tq, args, world, peaks):
    """One M=1 GEMV over the FFN gate/up projections stacked as one matrix:
    24 layers, [172032 x 1024], at G=128 (top-level keys) and G=64, four
    packed copies used in turn (154 and 165 MB, more than the 126 MB L2); and
    48 layers, [344064 x 1024], G=128, two copies (155 MB).  Launches run
    back to back from a CUDA graph: the streaming rate of the kernel with its
    per-launch fixed costs (grid-dependency wait, table build, cluster
    combine) included."""
    import torch
    K = 1024
    res = {}
    for layers, G, ncopy in [(24, 128, 4), (24, 64, 4), (48, 128, 2)]:
        N = layers * 2 * 3584
        packs = []
        for c in range(ncopy):
            W = device_weights(N, K, seed=77 + c)
            packs.append(tq.quantize_pack(W, G))
            del W
        torch.cuda.empty_cache()
        X = device_acts(1, K, seed=78)
        Y = torch.empty((1, N), dtype=torch.bfloat16, device="cuda")
        launches = [lambda c=c, s=s: tq.gemv(X, c, s, N, K, G, out=Y) for c, s in packs]
        us = graph_launch_us(launches, 16 // ncopy, args, world)
        byts = packed_bytes(N, K, G) + 2 * K + 2 * N
        gbs = byts / (us * 1e-6) / 1e9
        r = {"shape": [N, K], "G": G, "us": round(us, 2), "GB/s": round(gbs, 1),
             "frac": round(gbs / peaks["hbm_gbs"], 4), "launches": max(3, args.steps) * 16,
             "kernel": f"gemv_lut_stream_kernel<{G}, 3, 2> (lookup tables of one 512-column slice per CTA, "
                       "2-CTA clusters)",
             "note": f"{ncopy} copies of {byts / 1e6:.1f} MB used in turn from one CUDA graph "
                     f"({ncopy * byts / 1e6:.0f} MB > L2)"}
        if layers == 24 and G == 128:
            res.update(r)
            # 2 and 4 tokens on the same matrix (one streaming launch per token)
            for M in (2, 4):
                XM = device_acts(M, K, seed=79)
                YM = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
                lm = [lambda c=c, s=s: tq.gemv(XM, c, s, N, K, G, out=YM) for c, s in packs]
                usm = graph_launch_us(lm, 16 // ncopy, args, world)
                bm = packed_bytes(N, K, G) + 2 * M * K + 2 * M * N
                res[f"tokens{M}"] = {"us": round(usm, 2), "GB/s": round(bm / (usm * 1e-6) / 1e9, 1),
                                     "launches": max(3, args.steps) * 16 * M,
                                     "note": "one streaming launch per token; GB/s on the weights read once"}
                del lm, XM, YM
        else:
            res[f"stack{layers}_G{G}"] = r
        del packs, launches
        torch.cuda.empty_cache()
    return res


def decode_shapes_once(tq, args, world, peaks):
    """One tq_gemv launch (M=1) for each decode shape of the headline, gate
    3584x1024 and down 1024x3584 at both G, in that order: the run that the
    DRAM-traffic capture behind PREDECODE_DRAM_BYTES profiles (ncu flushes
    the caches before each profiled launch)."""
    import torch
    res = {}
    for G in GROUPS:
        for name in ("gate", "down"):
            N, K = FFN[name]
            c, s = tq.quantize_pack(device_weights(N, K, seed=7000), G)
            X = device_acts(1, K, seed=7100)
            tq.gemv(X, c, s, N, K, G)
            torch.cuda.synchronize()
            res[f"{name}{N}x{K}_G{G}"] = {"bytes": packed_bytes(N, K, G) + 2 * K + 2 * N}
    return res


def bench_gemv_shapes(tq, args, world, peaks):
    """Each decode projection alone (M=1, both G), and gate and up stacked as
    one [7168 x 1024] matrix (one launch for both): per-launch time over 160
    weight copies (130-275 MB, more than the 126 MB L2) replayed from a CUDA
    graph."""
    import torch
    res = {}
    shapes = [(n, nk) for n, nk in FFN.items() if n != "up"]
    shapes.append(("gateup", (2 * FFN["gate"][0], FFN["gate"][1])))  # gate and up stacked: one launch
    for G in GROUPS:
        for name, (N, K) in shapes:
            packs = []
            for c in range(160):
                W = device_weights(N, K, seed=7000 + c)
                packs.append(tq.quantize_pack(W, G))
                del W
            X = device_acts(1, K, seed=7100)
            Y = torch.empty((1, N), dtype=torch.bfloat16, device="cuda")
            for c, s in packs[:3]:
                tq.gemv(X, c, s, N, K, G, out=Y)
            torch.cuda.synchronize()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, capture_error_mode="relaxed"):
                for c, s in packs:
                    tq.gemv(X, c, s, N, K, G, out=Y)
            ms = timed(graph.replay, max(3, args.steps), max(3, args.warmup), world)
            us = ms * 1e3 / (max(3, args.steps) * len(packs))
            byts = packed_bytes(N, K, G) + 2 * K + 2 * N
            res[f"{name}{N}x{K}_G{G}"] = {"us": round(us, 2), "GB/s": round(byts / us / 1e3, 1),
                                           "launches": max(3, args.steps) * len(packs)}
            del packs
    return res


def bench_small_m_stack(tq, args, world, peaks):
    """5..64 tokens over the 24-layer gate/up stack as one [172032 x 1024]
    matrix, G=128 (the persistent small-M tensor kernel: more 128-row tiles
    than SMs): four packed copies (38.9 MB of codes and scales each, 156 MB
    in all, more than L2) used in turn from one CUDA graph.  GB/s on the
    algorithmic bytes (codes, scales, X, Y)."""
    import torch
    N, K, G = 48 * 3584, 1024, 128
    packs = []
    for c in range(4):
        W = device_weights(N, K, seed=77 + c)
        packs.append(tq.quantize_pack(W, G))
        del W
    torch.cuda.empty_cache()
    res = {}
    for M in (5, 16, 64):
        X = device_acts(M, K, seed=78)
        Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        launches = [lambda c=c, s=s: tq.gemv(X, c, s, N, K, G, out=Y) for c, s in packs]
        us = graph_launch_us(launches, 4, args, world)
        byts = packed_bytes(N, K, G) + 2 * M * K + 2 * M * N
        res[f"M{M}"] = {"us": round(us, 2), "GB/s": round(byts / us / 1e3, 1),
                        "frac": round(byts / us / 1e3 / peaks["hbm_gbs"], 4),
                        "TFLOP/s": round(2.0 * M * N * K / us / 1e6, 2), "launches": max(3, args.steps) * 16}
        del launches, X, Y
    res["kernel"] = "gemm_stream_kernel<NT, 3> (persistent, decoded W in tensor memory)"
    res["note"] = "4 copies of 38.9 MB used in turn from one CUDA graph (156 MB > L2)"
    del packs
    torch.cuda.empty_cache()
    return res


def bench_msweep(tq, args, world, peaks):
    """M-sweep over a 28-layer stack of q, o (1536x1536), gate, up (4096x1536)
    and down (1536x4096), G=128: one step = the 140 tq_gemv launches of one
    token batch of M rows, replayed from a CUDA graph (packed weights 144.5 MB,
    larger than L2).  Reports GB/s on the algorithmic bytes and TFLOP/s."""
    import torch
    G = 128
    packs = []
    for l in range(MSWEEP_LAYERS):
        for i, (name, (N, K)) in enumerate(MSWEEP.items()):
            W = device_weights(N, K, seed=9000 + 5 * l + i, outliers=False)
            packs.append((N, K) + tq.quantize_pack(W, G))
            del W
    wbytes = sum(packed_bytes(N, K, G) for (N, K, _, _) in packs)
    flops1 = sum(2 * N * K for (N, K, _, _) in packs)
    res = {}
    for M in MSWEEP_M:
        Xs = {K: device_acts(M, K, seed=9500 + K) for K in {k for (_, k, _, _) in packs}}
        Ys = {N: torch.empty((M, N), dtype=torch.bfloat16, device="cuda") for N in {n for (n, _, _, _) in packs}}

        def step():
            for (N, K, c, s_) in packs:
                tq.gemv(Xs[K], c, s_, N, K, G, out=Ys[N])
        step()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, capture_error_mode="relaxed"):
            step()
        steps = max(3, args.steps // 5)
        ms = timed(graph.replay, steps, max(3, args.warmup), world)
        us = ms * 1e3 / steps
        byts = wbytes + sum(2 * M * (K + N) for (N, K, _, _) in packs)
        gbs = byts / us / 1e3
        tfs = flops1 * M / us / 1e6
        bound = min(peaks["hbm_gbs"] * (flops1 * M / byts) / 1e3, peaks["bf16_tflops"])
        res[f"M{M}"] = {"us": round(us, 1), "GB/s": round(gbs, 1), "TFLOP/s": round(tfs, 2),
                        "frac_hbm": round(gbs / peaks["hbm_gbs"], 4), "roofline_TFLOP/s": round(bound, 1),
                        "frac_roofline": round(tfs / bound, 4), "launches": steps * len(packs)}
        del graph
    return res


def bench_bulk_codec(tq, args, world, peaks):
    """Quantize+pack and unpack over the 72-matrix FFN stack (24 layers), as two
    launches per direction: gate/up stacked [172032 x 1024] and downs [24576 x 3584]."""
    import torch
    shapes = [(48 * 3584, 1024), (24 * 1024, 3584)]
    out_pack, out_unpack = {}, {}
    for G in GROUPS:
        mats = [device_weights(N, K, seed=500 + i, outliers=False) for i, (N, K) in enumerate(shapes)]
        packed = [tq.quantize_pack(W, G) for W in mats]
        outs = [torch.empty_like(W) for W in mats]
        reps = max(3, args.steps // 4)

        def do_pack():  # into preallocated outputs, through the C ABI
            st = torch.cuda.current_stream().cuda_stream
            for W, (c, s) in zip(mats, packed):
                rc = tq.lib().tq_quantize_pack(W.data_ptr(), W.shape[0], W.shape[1], G,
                                               c.data_ptr(), s.data_ptr(), None, st)
                if rc != tq.TQ_OK:
                    raise tq.TQError(rc, "tq_quantize_pack")

        def do_unpack():
            for (c, s), o in zip(packed, outs):
                tq.unpack_bf16(c, s, o.shape[0], o.shape[1], G, out=o)

        ms_p = timed(do_pack, reps, max(3, args.warmup), world)
        ms_u = timed(do_unpack, reps, max(3, args.warmup), world)
        wbytes = sum(2 * N * K for N, K in shapes)
        pbytes = sum(packed_bytes(N, K, G) for N, K in shapes)
        for d, ms in ((out_pack, ms_p), (out_unpack, ms_u)):
            sec = ms * 1e-3 / reps
            d[f"G{G}"] = {"us": round(sec * 1e6, 1),
                          "packed_GB/s": round(pbytes / sec / 1e9, 1),
                          "total_GB/s": round((wbytes + pbytes) / sec / 1e9, 1),
                          "frac": round((wbytes + pbytes) / sec / 1e9 / peaks["hbm_gbs"], 4),
                          "launches": 2 * reps}
        del mats, packed, outs
        torch.cuda.empty_cache()
    return out_pack, out_unpack


def bench_ternary2(tq, args, world, peaks):
    """The 2-bit format (four codes per byte) through its own kernels:
    quantize + pack and unpack over the 72-matrix FFN stack, the streaming
    GEMV over the [172032 x 1024] gate/up stack (four copies, 187 MB > L2)
    and the decode chain of the headline (288 tq2_gemv launches, one graph)."""
    import torch
    res = {"pack": {}, "unpack": {}}
    shapes = [(48 * 3584, 1024), (24 * 1024, 3584)]
    reps = max(3, args.steps // 4)
    for G in GROUPS:
        mats = [device_weights(N, K, seed=500 + i, outliers=False) for i, (N, K) in enumerate(shapes)]
        packed = [tq.quantize_pack2(W, G) for W in mats]
        outs = [torch.empty_like(W) for W in mats]

        def do_pack():
            st = torch.cuda.current_stream().cuda_stream
            for W, (c, s) in zip(mats, packed):
                rc = tq.lib().tq2_quantize_pack(W.data_ptr(), W.shape[0], W.shape[1], G,
                                                c.data_ptr(), s.data_ptr(), None, st)
                if rc != tq.TQ_OK:
                    raise tq.TQError(rc, "tq2_quantize_pack")

        def do_unpack():
            for (c, s), o in zip(packed, outs):
                tq.unpack2_bf16(c, s, o.shape[0], o.shape[1], G, out=o)

        ms_p = timed(do_pack, reps, max(3, args.warmup), world)
        ms_u = timed(do_unpack, reps, max(3, args.warmup), world)
        wbytes = sum(2 * N * K for N, K in shapes)
        pbytes = sum(packed2_bytes(N, K, G) for N, K in shapes)
        for d, ms in ((res["pack"], ms_p), (res["unpack"], ms_u)):
            sec = ms * 1e-3 / reps
            d[f"G{G}"] = {"us": round(sec * 1e6, 1), "total_GB/s": round((wbytes + pbytes) / sec / 1e9, 1),
                          "frac": round((wbytes + pbytes) / sec / 1e9 / peaks["hbm_gbs"], 4),
                          "launches": 2 * reps}
        del mats, packed, outs
        torch.cuda.empty_cache()

    N, K, G = 48 * 3584, 1024, 128
    packs = []
    for c in range(4):
        W = device_weights(N, K, seed=77 + c)
        packs.append(tq.quantize_pack2(W, G))
        del W
    X = device_acts(1, K, seed=78)
    Y = torch.empty((1, N), dtype=torch.bfloat16, device="cuda")
    launches = [lambda c=c, s=s: tq.gemv2(X, c, s, N, K, G, out=Y) for c, s in packs]
    us = graph_launch_us(launches, 4, args, world)
    byts = packed2_bytes(N, K, G) + 2 * K + 2 * N
    gbs = byts / (us * 1e-6) / 1e9
    res["gemv_stream"] = {"shape": [N, K], "G": G, "us": round(us, 2), "GB/s": round(gbs, 1),
                          "frac": round(gbs / peaks["hbm_gbs"], 4), "launches": max(3, args.steps) * 16,
                          "kernel": "gemv_lut_stream_kernel<128, 2, 2> (lookup tables of 2-bit bytes, "
                                    "one 512-column slice per CTA)",
                          "note": "four copies used in turn from one CUDA graph"}
    del launches
    del packs
    torch.cuda.empty_cache()

    calls, _, Xs, Ys = build_decode_stack(tq, LAYERS, pack=None)
    packs2 = {}
    for G in GROUPS:
        for l in range(LAYERS):
            for i, (name, (N, K)) in enumerate(FFN.items()):
                W = device_weights(N, K, seed=1000 + 3 * l + i)
                packs2[(G, l, name)] = tq.quantize_pack2(W, G)
                del W
    step_bytes = sum(packed2_bytes(N, K, G) + 2 * K + 2 * N for (G, l, name, N, K, xo, yo) in calls)

    def step():
        for (G, l, name, N, K, xo, yo) in calls:
            c, s = packs2[(G, l, name)]
            tq.gemv2(Xs[xo:xo + K].view(1, K), c, s, N, K, G, out=Ys[yo:yo + N].view(1, N))
    step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, capture_error_mode="relaxed"):
        step()
    steps = max(3, args.steps // 5)
    ms = timed(graph.replay, steps, max(3, args.warmup), world)
    us = ms * 1e3 / steps
    res["decode_stack"] = {"launches_per_step": len(calls), "us_per_step": round(us, 1),
                           "us_per_launch": round(us / len(calls), 3), "GB/s": round(step_bytes / us / 1e3, 1),
                           "frac": round(step_bytes / us / 1e3 / peaks["hbm_gbs"], 4),
                           "launches": steps * len(calls), "bytes_per_step": step_bytes}
    del graph, packs2
    torch.cuda.empty_cache()

    # prefill on the tensor cores with 2-bit codes
    M, N, K = 4096, 14336, 4096
    W = device_weights(N, K, seed=904, outliers=False)
    c2, s2 = tq.quantize_pack2(W, 128)
    del W
    X = device_acts(M, K, seed=905)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    tq.gemm2(X, c2, s2, N, K, 128, out=Y)
    preps = max(3, args.steps // 4)
    ms = timed_flushed(lambda: tq.gemm2(X, c2, s2, N, K, 128, out=Y), preps, max(3, args.warmup), world)
    tflops = 2.0 * M * N * K * preps / (ms * 1e-3) / 1e12
    res["prefill"] = {"M": M, "N": N, "K": K, "G": 128, "us": round(ms * 1e3 / preps, 1),
                      "TFLOP/s": round(tflops, 1), "frac": round(tflops / peaks["bf16_tflops"], 4), "launches": preps}
    del c2, s2, X, Y
    torch.cuda.empty_cache()
    return res


def device_w4_params(N, K, G, seed):
    """Seeded W4A16 parameters made on the device: uniform 4-bit codes, scale
    magnitudes 0.004..0.009 with random signs, biases ~ N(0, 0.05) (an affine
    4-bit quantization of N(0, 0.02) weights over groups of G)."""
    import torch
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    codes = torch.randint(-(1 << 31), (1 << 31) - 1, (N, K // 8), generator=g, device="cuda", dtype=torch.int64)
    codes = codes.to(torch.int32)
    mag = torch.rand((N, K // G), generator=g, device="cuda") * 0.005 + 0.004
    sign = torch.where(torch.rand((N, K // G), generator=g, device="cuda") < 0.5, -1.0, 1.0)
    scales = (mag * sign).to(torch.bfloat16)
    biases = (torch.randn((N, K // G), generator=g, device="cuda") * 0.05).to(torch.bfloat16)
    return codes, scales, biases


def w4_bytes(N, K, G):
    return N * K // 2 + 4 * N * (K // G)


def bench_w4(tq, args, world, peaks):
    """The W4A16 affine format (the second weight format): the streaming
    decode GEMV over the [172032 x 1024] gate/up-shaped stack at G=128 (four
    copies, 374 MB > L2, used in turn from one CUDA graph) and the
    tensor-core prefill GEMM at M=4096, 4096 -> 14336 (L2 flushed before
    every launch)."""
    import torch
    res = {}
    N, K, G = 48 * 3584, 1024, 128
    ncopy = 4
    packs = [device_w4_params(N, K, G, seed=300 + c) for c in range(ncopy)]
    X = device_acts(1, K, seed=301)
    Y = torch.empty((1, N), dtype=torch.bfloat16, device="cuda")
    launches = [lambda p=p: tq.w4_gemv(X, p[0], p[1], p[2], N, K, G, out=Y) for p in packs]
    us = graph_launch_us(launches, 16 // ncopy, args, world)
    byts = w4_bytes(N, K, G) + 2 * K + 2 * N
    gbs = byts / (us * 1e-6) / 1e9
    res["gemv_stream"] = {"shape": [N, K], "G": G, "us": round(us, 2), "GB/s": round(gbs, 1),
                          "frac": round(gbs / peaks["hbm_gbs"], 4), "launches": max(3, args.steps) * 16,
                          "kernel": "gemv_lut_stream_kernel<128, 4, 4> (lookup tables of one 256-column slice "
                                    "per CTA, 4-CTA clusters)",
                          "note": f"{ncopy} copies of {byts / 1e6:.1f} MB used in turn from one CUDA graph"}
    del packs, launches
    torch.cuda.empty_cache()
    M, N, K = 4096, 14336, 4096
    c, s_, b = device_w4_params(N, K, G, seed=302)
    X = device_acts(M, K, seed=303)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    tq.w4_gemm(X, c, s_, b, N, K, G, out=Y)
    preps = max(3, args.steps // 4)
    ms = timed_flushed(lambda: tq.w4_gemm(X, c, s_, b, N, K, G, out=Y), preps, max(3, args.warmup), world)
    tflops = 2.0 * M * N * K * preps / (ms * 1e-3) / 1e12
    res["prefill"] = {"M": M, "N": N, "K": K, "G": G, "us": round(ms * 1e3 / preps, 1), "TFLOP/s": round(tflops, 1),
                      "frac": round(tflops / peaks["bf16_tflops"], 4), "launches": preps,
                      "note": "each weight as two bf16 terms: two MMAs per product, so at most half the bf16 rate"}
    del c, s_, b, X, Y
    torch.cuda.empty_cache()
    return res


def bench_prefill(tq, args, world, peaks):
    import torch
    M, G = 4096, 128
    res = {}
    for name, (N, K) in (("up", (14336, 4096)), ("down", (4096, 14336))):
        W = device_weights(N, K, seed=900 + len(res), outliers=False)
        codes, scales = tq.quantize_pack(W, G)
        del W
        X = device_acts(M, K, seed=950 + len(res))
        Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        try:
            tq.gemm(X, codes, scales, N, K, G, out=Y)
        except tq.TQError as e:
            res[name] = {"unavailable": str(e)}
            continue
        reps = max(3, args.steps // 4)
        ms = timed_flushed(lambda: tq.gemm(X, codes, scales, N, K, G, out=Y), reps, max(3, args.warmup), world)
        tflops = 2.0 * M * N * K * reps / (ms * 1e-3) / 1e12
        res[name] = {"M": M, "N": N, "K": K, "G": G, "us": round(ms * 1e3 / reps, 1),
                     "TFLOP/s": round(tflops, 1), "frac": round(tflops / peaks["bf16_tflops"], 4),
                     "launches": reps, "l2": "flushed before every launch (256 MB write, outside the events)"}
    return res


# --------------------------------------------------------------------- oracle (CPU)

_ORACLE_MATS = None


def oracle_mats():
    """Layer-0 gate, up and down projections packed by the oracle for G=64
    and G=128, with their M=1 activations (prepared outside any timing)."""
    global _ORACLE_MATS
    if _ORACLE_MATS is None:
        import oracle
        import synthetic
        mats = []
        for G in GROUPS:
            for name in ("gate", "up", "down"):
                W = synthetic.ffn_matrix(name)
                N, K = W.shape
                codes, scales, _ = oracle.quantize_pack(W, G)
                mats.append((synthetic.activations(1, K), codes, scales, N, K, G))
        _ORACLE_MATS = mats
    return _ORACLE_MATS


def oracle_sample_step():
    """One bounded sample of the decode workload on the CPU oracle: decode
    GEMV (decode to bf16 + binary64 matmul) of the layer-0 gate, up and down
    projections for G=64 and G=128 at M=1.  Returns the algorithmic bytes."""
    import oracle
    nbytes = 0
    for X, codes, scales, N, K, G in oracle_mats():
        oracle.linear(X, codes, scales, N, K, G)
        nbytes += packed_bytes(N, K, G) + 2 * K + 2 * N
    return nbytes


def _oracle_pool_init(mats):
    global _ORACLE_MATS
    _ORACLE_MATS = mats


def _oracle_rows_pass(job):
    """Worker: decode GEMV (decode to bf16 + binary64 matmul) of rows
    [N*part/nparts, N*(part+1)/nparts) of every sampled matrix."""
    import oracle
    part, nparts = job
    for X, codes, scales, N, K, G in _ORACLE_MATS:
        lo, hi = N * part // nparts, N * (part + 1) // nparts
        if hi > lo:
            oracle.linear(X, codes[lo:hi], scales[lo:hi], hi - lo, K, G)
    return part


class OraclePool:
    """The single-threaded C oracle run by one spawned process per host CPU
    (rows split evenly), for the all-core baseline.  Spawned, not forked, so
    no child inherits a CUDA context."""

    def __init__(self, n=None):
        import multiprocessing as mp
        self.n = n or host_cpu()["affinity_cpus"] or 1
        self.pool = mp.get_context("spawn").Pool(self.n, initializer=_oracle_pool_init,
                                                  initargs=(oracle_mats(),))
        self.jobs = [(i, self.n) for i in range(self.n)]
        self.pool.map(_oracle_rows_pass, self.jobs)  # workers up and warm

    def step(self):
        """One pass over the whole sample; returns its algorithmic bytes."""
        self.pool.map(_oracle_rows_pass, self.jobs)
        return sum(packed_bytes(N, K, G) + 2 * K + 2 * N for (_, _, _, N, K, G) in oracle_mats())

    def close(self):
        self.pool.close()
        self.pool.join()


def _timed_passes(step, budget_s):
    t0 = time.perf_counter()
    nbytes = reps = 0
    while True:
        nbytes += step()
        reps += 1
        if time.perf_counter() - t0 > budget_s:
            break
    return nbytes, reps, time.perf_counter() - t0


SAMPLE_DESC = "decode GEMV (decode to bf16 + binary64 matmul) over layer-0 gate/up/down for G=64 and G=128, M=1"


def cpu_baseline(args, budget_s=10.0):
    """The oracle as it stands (plain C, binary64) timed on this host on a
    bounded sample -- repeated decode GEMVs of the layer-0 projections --
    on every host CPU (one spawned process per CPU, rows split) and on one."""
    oracle_mats()
    host = host_cpu()
    pool = OraclePool()
    try:
        nb, reps, sec = _timed_passes(pool.step, budget_s)
    finally:
        pool.close()
    nb1, reps1, sec1 = _timed_passes(oracle_sample_step, budget_s)
    return {"value": round(nb / sec / 1e9, 4), "unit": "GB/s", "cores": pool.n, "kind": "oracle",
            "sample": f"{reps} passes of the {SAMPLE_DESC}, rows split over {pool.n} processes, {sec:.1f} s",
            "host": host,
            "single_thread": {"value": round(nb1 / sec1 / 1e9, 4), "unit": "GB/s", "cores": 1,
                              "sample": f"{reps1} passes of the same sample, {sec1:.1f} s"}}


def run_reference(args, rank, world):
    if rank != 0:
        return
    t = []
    nbytes = 0
    oracle_mats()
    pool = OraclePool()
    try:
        for _ in range(args.warmup):
            pool.step()
        for _ in range(args.steps):
            t0 = time.perf_counter()
            nbytes = pool.step()
            t.append(time.perf_counter() - t0)
    finally:
        pool.close()
    total = sum(t)
    value = nbytes * len(t) / total / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * total / len(t), 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "decode GEMV, M=1, Qwen3.5-0.8B-shaped FFN gate/up 3584x1024 and "
                               "down 1024x3584, G in {64,128}; each step a bounded sample: layer 0's "
                               "three projections for both G (decode to bf16 + binary64 matmul)"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": pool.n, "kind": "oracle",
                         "sample": f"layer-0 gate/up/down, G=64 and 128, M=1, per step, rows split over "
                                   f"{pool.n} spawned processes", "host": host_cpu()},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["tq", "reference"], default="tq")
    ap.add_argument("--only", choices=["stream", "codec", "prefill", "gemv", "msweep", "smallm", "ternary2", "w4",
                                       "traffic"],
                    default=None,
                    help="run one sub-benchmark alone and print its result (profiling aid)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":  # CPU only: rank 0 runs, the others exit without work
        run_reference(args, int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")))
        return
    rank, world, local = dist_setup(args)
    try:
        if args.only:
            import torch
            import ternary_weight_only_group_b200 as tq
            torch.cuda.set_device(local)
            peaks = load_peaks()
            fn = {"stream": bench_gemv_stream, "codec": bench_bulk_codec, "prefill": bench_prefill,
                  "gemv": bench_gemv_shapes, "msweep": bench_msweep, "smallm": bench_small_m_stack,
                  "ternary2": bench_ternary2, "w4": bench_w4,
                  "traffic": decode_shapes_once}
            res = fn[args.only](tq, args, world, peaks)
            if rank == 0:
                print(json.dumps({"only": args.only, "result": res}), flush=True)
            return
        run_ours(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            if dist.is_initialized():
                dist.destroy_process_group()


if __name__ == "__main__":
    main()
