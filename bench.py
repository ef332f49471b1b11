#!/usr/bin/env python
"""Benchmark: batch-1 INT4 fused-dequant GEMV over a Llama-7B-shaped decode stack.

Workload (one "step" = one decode token through the stack's linear layers):
  32 layers x {qkv 4096->12288, o 4096->4096, gate 4096->11008, up 4096->11008,
  down 11008->4096}, INT4 asymmetric RTN, group 128, batch 1, fp16 activations
  x ~ N(0, 1), weights W = 0.02 * t5 * lognormal_row(0, 0.5) drawn on the GPU
  with a seeded generator and quantized by qnt_quantize.  160 GEMVs per step,
  3.37 GB of packed weights per step: larger than L2, so every step reads its
  weights from HBM (no flush needed).

The step is one qnt_gemv_seq call (one persistent kernel for the 160 GEMVs);
every GEMV is marked `wait`, so it reads its x only after the previous GEMV of
the step has written its y, as if x were computed from it.  Also reported: the
same 160 GEMVs as separate qnt_gemv launches (programmatic dependent launch,
captured in a CUDA graph), and each layer shape alone.

Metric: achieved HBM GB/s from algorithmic bytes (codes + metadata + x + y per
GEMV) and microseconds per decode layer (step time / 32).  Timing uses CUDA
events on the launching stream, with a barrier and synchronize around the timed
region and the max over ranks for N > 1 (each rank runs its own replica: weak
scaling).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

LAYERS = 32
HIDDEN, INTER, QKV = 4096, 11008, 12288
SHAPES = [("qkv", QKV, HIDDEN), ("o", HIDDEN, HIDDEN), ("gate", INTER, HIDDEN), ("up", INTER, HIDDEN),
          ("down", HIDDEN, INTER)]   # (name, N, K)
GROUP = 128
WORKLOAD = "llama7b_decode_stack_int4_g128_b1"
METRIC = "4-bit fused-dequant GEMV HBM GB/s (% of peak) and us per decode layer"


def algo_bytes_int4(N, K, g=GROUP, M=1):
    """Algorithmic bytes of one INT4 GEMV: 4-bit codes, fp16 scale + 4-bit zero
    per group, fp16 x and y."""
    return N * K // 2 + (N * K // g) * 5 // 2 + 2 * K * M + 2 * N * M


STEP_BYTES = LAYERS * sum(algo_bytes_int4(N, K) for _, N, K in SHAPES)
# DRAM bytes (read + write) of one launch of the sequence kernel over the whole
# stack: an ncu capture of one decode layer (`--kernel-only layer`, 105.24 MB
# read + 3.65 MB written, the kernel as built now) times the 32 layers, which
# stream the same shapes.  None when the kernel has changed since the capture.
TRAFFIC_PER_LAUNCH = 3_484_631_040


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d.get("hbm_gbs", 6650.0), "measured"
    return 6650.0, "fallback"


def measured_tensor_peak():
    """bf16 dense TFLOP/s measured by a seconds-long cuBLAS loop (sustained)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        if "bf16_tflops_sustained" in d:
            return d["bf16_tflops_sustained"], "measured (sustained)"
    return 1400.0, "fallback (sustained)"


META_BYTES_PER_GROUP = {1: 2.5, 2: 2.0, 3: 4.0, 4: 2.25}   # INT4, FP4, AFPQ, RaZeR


def algo_bytes(fmt, N, K, M, g=GROUP):
    """Algorithmic bytes of one GEMV / GEMM: codes + metadata + activations + outputs."""
    if fmt == 5:                      # INT8 per channel: a byte per weight, an fp16 scale per row
        wbytes = N * K + 2 * N
    elif fmt == 6:                    # FP16
        wbytes = 2 * N * K
    else:
        wbytes = N * K // 2 + int(N * K // g * META_BYTES_PER_GROUP[fmt])
    return wbytes + 2 * K * M + 2 * N * M


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.samples = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), [x.strip() for x in line.split(",")]))

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0, t1):
        win = [s for t, s in self.samples if t0 - 0.15 <= t <= t1 + 0.15]
        if not win and self.samples:
            mid = 0.5 * (t0 + t1)
            win = [min(self.samples, key=lambda ts: abs(ts[0] - mid))[1]]
        if not win:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        sm = [float(s[1]) for s in win if s[1].replace(".", "").isdigit()]
        mx = [float(s[2]) for s in win if s[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for s in win for i in range(4) if len(s) > 5 + i and s[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(win)}


# ------------------------------------------------------------------ distributed plumbing
def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def allreduce_max(v, world):
    """Max of a host float over the ranks (a timing: the slowest rank decides)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_value(step_bytes, world, step_ms):
    """Whole-job GB/s of `world` independent replicas that each stream
    step_bytes per step; step_ms is the step time, max over the ranks."""
    return world * step_bytes / (step_ms * 1e-3) / 1e9


# ------------------------------------------------------------------ our arm
def build_stack(Q, torch, seed_base):
    """Quantize 32 layers of Llama-7B-shaped weights on the GPU."""
    from dequant_gemv_rtn_b200 import synth
    layers = []
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    for l in range(LAYERS):
        mods = []
        for mi, (name, N, K) in enumerate(SHAPES):
            d = Q.desc(Q.QNT_INT4_ASYM, N, K, GROUP)
            W = synth.llama_like_device(N, K, seed=seed_base + 16 * l + mi)
            codes = torch.empty(Q.qnt_codes_bytes(d), dtype=torch.uint8, device="cuda")
            meta = torch.empty(Q.qnt_meta_bytes(d), dtype=torch.uint8, device="cuda")
            Q.qnt_quantize(d, W, codes, meta, st)
            del W
            mods.append((name, d, codes, meta))
        layers.append(mods)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, f"quantize status {int(st.item())}"
    return layers


def run_ours(args, world, rank, local):
    import torch
    from dequant_gemv_rtn_b200 import qnt as Q
    from dequant_gemv_rtn_b200 import synth
    torch.cuda.set_device(local)
    dev_index = torch.cuda.current_device()
    layers = build_stack(Q, torch, seed_base=1000 * (rank + 1))
    xs = {K: synth.activations_device(1, K, seed=7 + K, dtype=torch.float16) for K in (HIDDEN, INTER)}
    ys = {(name, l): torch.empty(N, dtype=torch.float16, device="cuda")
          for l in range(LAYERS) for name, N, _ in SHAPES}
    stream = torch.cuda.Stream()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")

    # decode-layer dependencies: each GEMV reads its x after the GEMV that
    # produces it (o <- qkv, gate <- o, up <- o, down <- up and gate, the next
    # layer's qkv <- down); as steps back in the sequence:
    layer_wait = {"qkv": 1, "o": 1, "gate": 1, "up": 2, "down": 1}

    def seq_items(x_of, y_of, waits=None):
        return [(d, codes, meta, x_of(l, name, d), y_of(l, name),
                 (waits or layer_wait)[name] if (l, name) != (0, "qkv") else 0)
                for l, mods in enumerate(layers) for name, d, codes, meta in mods]

    steps = Q.seq_steps(seq_items(lambda l, name, d: xs[d.K], lambda l, name: ys[(name, l)]))
    serial = Q.seq_steps(seq_items(lambda l, name, d: xs[d.K], lambda l, name: ys[(name, l)],
                                   {n: 1 for n in layer_wait}))
    work = torch.zeros(Q.qnt_gemv_seq_work_bytes(len(steps)), dtype=torch.uint8, device="cuda")

    def step_seq(s):
        Q.qnt_gemv_seq(steps, Q.QNT_F16, work, st, s)

    def step_serial(s):
        Q.qnt_gemv_seq(serial, Q.QNT_F16, work, st, s)

    def step_launches(s):
        for l, mods in enumerate(layers):
            for name, d, codes, meta in mods:
                Q.qnt_gemv(d, codes, meta, xs[d.K], ys[(name, l)], Q.QNT_F16, st, s)

    graphs = []   # every captured graph lives until the end of the run

    def time_graph(run, reps):
        with torch.cuda.stream(stream):
            run(stream)               # eager first (per-kernel attributes are set outside capture)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            run(torch.cuda.current_stream())
        graphs.append(g)
        for _ in range(args.warmup):
            g.replay()
        torch.cuda.synchronize()
        per = []
        with torch.cuda.stream(stream):
            for _ in range(reps):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                g.replay()
                e1.record(stream)
                per.append((e0, e1))
        torch.cuda.synchronize()
        return g, [x.elapsed_time(y) for x, y in per]

    # headline: the sequence kernel, one launch per step
    graph, _ = time_graph(step_seq, 1)
    sampler = ClockSampler(dev_index)
    sampler.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = time.time()
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    t1 = time.time()
    barrier(world)
    sampler.stop()
    ms = e0.elapsed_time(e1)
    ms = allreduce_max(ms, world)
    clocks = sampler.summary(t0, t1)
    assert int(st.item()) == 0, f"device status {int(st.item())}"
    # per-step distribution (separately timed replays)
    _, seq_ms = time_graph(step_seq, max(10, min(args.steps, 200)))
    # every GEMV waiting for the one before it
    _, serial_ms = time_graph(step_serial, max(10, min(args.steps, 100)))
    # the same GEMVs as separate launches (qnt_gemv, programmatic dependent launch)
    _, chain_ms = time_graph(step_launches, max(10, min(args.steps, 100)))

    pct = lambda v, q: float(np.percentile(v, q))
    # per-shape isolated launch times (same kernel, 32 cold layers per graph)
    per_shape = {}
    for mi, (name, N, K) in enumerate(SHAPES):
        def shape_launches(s, mi=mi, name=name, K=K):
            for l in range(LAYERS):
                _, d, codes, meta = layers[l][mi]
                Q.qnt_gemv(d, codes, meta, xs[K], ys[(name, l)], Q.QNT_F16, st, s)
        _, shape_ms = time_graph(shape_launches, 20)
        us = statistics.median(shape_ms) * 1000.0 / LAYERS
        per_shape[f"{name}_{K}x{N}"] = {"us": round(us, 3), "GBps": round(algo_bytes_int4(N, K) / us / 1e3, 1),
                                        "p10_p90_us": [round(pct(shape_ms, 10) * 1000.0 / LAYERS, 3),
                                                       round(pct(shape_ms, 90) * 1000.0 / LAYERS, 3)]}

    # end to end through the public API with host buffers: per step, the step's
    # inputs (every GEMV's x, one pinned host buffer) go host->device in one copy
    # and the step's results (every y) come back device->host in one copy
    x_off, y_off, nx, ny = {}, {}, 0, 0
    for l in range(LAYERS):
        for name, N, K in SHAPES:
            x_off[(name, l)], y_off[(name, l)] = (nx, K), (ny, N)
            nx, ny = nx + K, ny + N
    h_in = torch.empty(nx, dtype=torch.float16).pin_memory()
    for (name, l), (o, K) in x_off.items():
        h_in[o:o + K].copy_(xs[K].reshape(-1).cpu())
    d_in = torch.empty(nx, dtype=torch.float16, device="cuda")
    d_out = torch.empty(ny, dtype=torch.float16, device="cuda")
    h_out = torch.empty(ny, dtype=torch.float16).pin_memory()

    e2e_steps_desc = Q.seq_steps(seq_items(lambda l, name, d: d_in[x_off[(name, l)][0]:x_off[(name, l)][0] + d.K],
                                           lambda l, name: d_out[y_off[(name, l)][0]:y_off[(name, l)][0] + y_off[(name, l)][1]]))

    def e2e_step(s):
        d_in.copy_(h_in, non_blocking=True)
        Q.qnt_gemv_seq(e2e_steps_desc, Q.QNT_F16, work, st, s)
        h_out.copy_(d_out, non_blocking=True)

    with torch.cuda.stream(stream):
        e2e_step(stream)
    torch.cuda.synchronize()
    ge = torch.cuda.CUDAGraph()
    with torch.cuda.graph(ge, stream=stream):
        e2e_step(torch.cuda.current_stream())
    for _ in range(max(3, args.warmup)):
        ge.replay()
    torch.cuda.synchronize()
    barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_steps = max(1, min(args.steps, 200))
    with torch.cuda.stream(stream):
        a.record(stream)
        for _ in range(e2e_steps):
            ge.replay()
        b.record(stream)
    torch.cuda.synchronize()
    e2e_ms = allreduce_max(a.elapsed_time(b), world) / e2e_steps
    h2d = LAYERS * sum(2 * K for _, _, K in SHAPES)
    d2h = LAYERS * sum(2 * N for _, N, _ in SHAPES)
    del ge
    torch.cuda.synchronize()
    graphs.clear()

    step_ms = ms / args.steps
    value = replica_value(STEP_BYTES, world, step_ms)
    peak, peak_kind = measured_peaks()
    result = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(step_ms, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int4 weights, fp16 activations, fp32 accumulate", "data": "synthetic",
        "config": {"workload": WORKLOAD, "layers": LAYERS, "shapes_NxK": [[N, K] for _, N, K in SHAPES],
                   "group": GROUP, "batch": 1, "bytes_per_step": STEP_BYTES,
                   "l2": "inputs larger than L2 (3.37 GB of packed weights per step), no flush",
                   "timing": "CUDA graph of one step (one qnt_gemv_seq call) replayed; CUDA events on the "
                             "launching stream",
                   "dependencies": "decode-layer order: each GEMV reads its x after the GEMV that produces it "
                                   "(o<-qkv, gate<-o, up<-o, down<-gate,up, next qkv<-down)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "us_per_layer": round(step_ms * 1000.0 / LAYERS, 3),
        "us_per_layer_p10_p90": [round(pct(seq_ms, 10) * 1000.0 / LAYERS, 3),
                                 round(pct(seq_ms, 90) * 1000.0 / LAYERS, 3)],
        "roofline": {"bound": "hbm", "achieved": round(STEP_BYTES / (step_ms * 1e-3) / 1e9, 1),
                     "peak": peak, "peak_kind": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs, copy)" if peak_kind == "measured" else "fallback",
                     "unit": "GB/s", "frac": round(STEP_BYTES / (step_ms * 1e-3) / 1e9 / peak, 4),
                     "traffic": TRAFFIC_PER_LAUNCH, "kernel": "gemv1_kernel<INT4,g128> (sequence of 160 GEMVs)",
                     "per_launch_bytes": STEP_BYTES, "launches_per_step": 1},
        "serialized": {"us_per_layer": round(statistics.median(serial_ms) * 1000.0 / LAYERS, 3),
                       "GBps": round(STEP_BYTES / (statistics.median(serial_ms) * 1e-3) / 1e9, 1),
                       "how": "qnt_gemv_seq with every GEMV waiting for the one before it; median of replays"},
        "per_launch_chain": {"us_per_layer": round(statistics.median(chain_ms) * 1000.0 / LAYERS, 3),
                             "GBps": round(STEP_BYTES / (statistics.median(chain_ms) * 1e-3) / 1e9, 1),
                             "how": "the same 160 GEMVs as qnt_gemv launches (programmatic dependent launch) "
                                    "in one CUDA graph; median of replays"},
        "per_shape_isolated": per_shape,
        "gpu_launches": args.steps,
        "clocks": clocks,
        "e2e": {"value": round(replica_value(STEP_BYTES, world, e2e_ms), 1), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "how": "public C-ABI qnt_gemv_seq; per step, every GEMV's x copied host->device from one pinned "
                       "buffer and every y copied back in one device->host copy, inside a captured CUDA graph; "
                       "weights resident"},
    }
    return result, layers


# ------------------------------------------------------------------ CPU oracle (baseline / reference arm)
def oracle_layer(torch, seed_base=1000):
    """One decode layer's weights drawn on the GPU, copied to the host and
    quantized by the oracle (timed separately from the GEMV)."""
    from dequant_gemv_rtn_b200 import synth
    from oracle import oracle as orc
    mods = []
    for mi, (name, N, K) in enumerate(SHAPES):
        W = synth.llama_like_device(N, K, seed=seed_base + mi).cpu().numpy()
        q = orc.quantize(orc.INT4, W, GROUP)
        del W
        x = orc.f2h(synth.activations(1, K, seed=7 + K))
        mods.append((q, x))
    return mods


def time_oracle_layer(mods, budget_s):
    from oracle import oracle as orc
    t0 = time.perf_counter()
    n = 0
    while True:
        for q, x in mods:
            orc.gemm(q, x, 0)
        n += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    return (time.perf_counter() - t0) / n, n


def cpu_baseline(torch, budget_s=10.0):
    from oracle import oracle as orc
    mods = oracle_layer(torch)
    per_layer_s, n = time_oracle_layer(mods, budget_s)
    layer_bytes = sum(algo_bytes_int4(N, K) for _, N, K in SHAPES)
    return {"value": round(layer_bytes / per_layer_s / 1e9, 3), "unit": "GB/s", "cores": orc.threads(),
            "kind": "oracle",
            "sample": f"{n} pass(es) of the oracle's binary64 GEMV over one of the 32 decode layers "
                      f"(5 INT4 g128 matrices, {layer_bytes} algorithmic bytes); {per_layer_s * 1e3:.1f} ms per layer"}


def run_reference(args, world, rank, local):
    import torch
    if rank != 0:
        return None
    torch.cuda.set_device(local)
    from oracle import oracle as orc
    mods = oracle_layer(torch)
    layer_bytes = sum(algo_bytes_int4(N, K) for _, N, K in SHAPES)
    for _ in range(args.warmup):
        for q, x in mods:
            orc.gemm(q, x, 0)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        for q, x in mods:
            orc.gemm(q, x, 0)
    per_step = (time.perf_counter() - t0) / args.steps
    value = layer_bytes / per_step / 1e9
    sample = (f"each step = the oracle's binary64 GEMV over one decode layer (5 INT4 g128 matrices of the "
              f"{LAYERS}-layer stack)")
    return {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(per_step * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 accumulate",
            "data": "synthetic", "config": {"workload": WORKLOAD, "layers_per_step": 1, "group": GROUP, "batch": 1},
            "us_per_layer": round(per_step * 1e6, 1),
            "cpu_baseline": {"value": round(value, 3), "unit": "GB/s", "cores": orc.threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 3), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ------------------------------------------------------------------ the other workloads
def _time_graph(torch, stream, run, warmup, reps):
    """Capture run(stream) in a CUDA graph, replay; per-replay ms (CUDA events)."""
    with torch.cuda.stream(stream):
        run(stream)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        run(torch.cuda.current_stream())
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    ev = []
    with torch.cuda.stream(stream):
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            g.replay()
            b.record(stream)
            ev.append((a, b))
    torch.cuda.synchronize()
    out = [a.elapsed_time(b) for a, b in ev]
    del g
    return out


def _quantized(Q, torch, synth, fmt, N, K, g, seed, st):
    d = Q.desc(fmt, N, K, g)
    W = synth.llama_like_device(N, K, seed=seed)
    codes = torch.empty(Q.qnt_codes_bytes(d), dtype=torch.uint8, device="cuda")
    meta = torch.empty(max(16, Q.qnt_meta_bytes(d)), dtype=torch.uint8, device="cuda")
    Q.qnt_quantize(d, W, codes, meta, st)
    del W
    return d, codes, meta


def run_extra_configs(args):
    """The pages' other workloads, each in the launch configuration its parity
    test covers: FP4 / AFPQ / RaZeR on K=4096, N=14336 at batch 1 and 4; the
    Llama-70B INT4 GEMMs at M = 1..128 with bf16 activations; the
    selective-precision Llama-2-7B stack at batch 1 and 16.  Each matrix is
    timed over enough rotating copies that its weights come from HBM."""
    import torch
    from dequant_gemv_rtn_b200 import qnt as Q
    from dequant_gemv_rtn_b200 import synth
    hbm, hbm_kind = measured_peaks()
    tpeak, tkind = measured_tensor_peak()
    stream = torch.cuda.Stream()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    pct = lambda v, q: float(np.percentile(v, q))
    reps = 20
    out = {"peaks": {"hbm_GBps": hbm, "hbm_kind": hbm_kind, "bf16_TFLOPs": tpeak, "bf16_kind": tkind}}

    def timed(name, fmt, N, K, M, xdt, copies):
        """copies: list of (d, codes, meta); times qnt_gemv (M = 1) or qnt_gemm."""
        X = synth.activations_device(M, K, seed=11, dtype=torch.bfloat16 if xdt else torch.float16)
        Y = torch.empty((M, N), dtype=X.dtype, device="cuda")

        def run(s):
            for d, c, m in copies:
                if M == 1:
                    Q.qnt_gemv(d, c, m, X, Y, xdt, st, s)
                else:
                    Q.qnt_gemm(d, c, m, X, Y, M, xdt, st, s)
        ms = _time_graph(torch, stream, run, 3, reps)
        us = [t * 1000.0 / len(copies) for t in ms]
        med = statistics.median(us)
        byts = algo_bytes(fmt, N, K, M)
        r = {"us": round(med, 3), "p10_p90_us": [round(pct(us, 10), 3), round(pct(us, 90), 3)],
             "GBps": round(byts / med / 1e3, 1), "frac_hbm": round(byts / med / 1e3 / hbm, 4)}
        if M > 1:
            tfl = 2.0 * M * N * K / med / 1e6
            r["TFLOPs"] = round(tfl, 1)
            r["frac_tensor"] = round(tfl / tpeak, 4)
        assert int(st.item()) == 0, f"{name}: device status {int(st.item())}"
        return r

    def ncopies(nbytes):
        return max(2, min(8, int(4 * 126e6 // max(nbytes, 1)) + 1))

    # FP4 family, K=4096 N=14336, batch 1 and 4 (fp16 activations)
    for fmt, fname in ((2, "fp4"), (3, "afpq"), (4, "razer")):
        N, K = 14336, 4096
        copies = [_quantized(Q, torch, synth, fmt, N, K, GROUP, 40 + i, st) for i in range(ncopies(algo_bytes(fmt, N, K, 1)))]
        for M in (1, 2, 4, 8):
            out[f"{fname}_g128_{K}x{N}_b{M}"] = timed(fname, fmt, N, K, M, 0, copies)
        del copies
        torch.cuda.empty_cache()
    # Llama-70B INT4 g128, bf16 activations, M sweep
    for N, K in ((10240, 8192), (28672, 8192), (8192, 28672)):
        copies = [_quantized(Q, torch, synth, 1, N, K, GROUP, 60 + i, st) for i in range(ncopies(algo_bytes(1, N, K, 1)))]
        for M in (1, 2, 4, 8, 16, 32, 64, 128):
            out[f"int4_g128_{K}x{N}_bf16_M{M}"] = timed("llama70b", 1, N, K, M, 1, copies)
        del copies
        torch.cuda.empty_cache()
    # selective-precision Llama-2-7B stack: INT4 g128, INT8 per channel for
    # down_proj of layers 0, 1, 30, 31, FP16 lm_head; batch 1 and 16
    t = Q.qnt_table_create(Q.QNT_INT4_ASYM, GROUP)
    for layer in (0, 1, 30, 31):
        t.set(f"layers.{layer}.mlp.down_proj", Q.QNT_INT8_PERCHAN, 0)
    t.set("lm_head", Q.QNT_FP16, 0)
    mods = []
    for l in range(32):
        mods += [(f"layers.{l}.self_attn.{p}", 4096, 4096) for p in ("q_proj", "k_proj", "v_proj", "o_proj")]
        mods += [(f"layers.{l}.mlp.gate_proj", 11008, 4096), (f"layers.{l}.mlp.up_proj", 11008, 4096),
                 (f"layers.{l}.mlp.down_proj", 4096, 11008)]
    stack, stack_bytes = [], {1: 0, 16: 0}
    for i, (name, N, K) in enumerate(mods):
        fmt, g = t.lookup(name)
        stack.append((fmt, N, K) + _quantized(Q, torch, synth, fmt, N, K, g if g else K, 900 + i, st))
        for M in (1, 16):
            stack_bytes[M] += algo_bytes(fmt, N, K, M)
    head = _quantized(Q, torch, synth, Q.QNT_FP16, 32000, 4096, 4096, 899, st)
    t.close()
    for M in (1, 16):
        Xs = {K: synth.activations_device(M, K, seed=K, dtype=torch.float16) for K in (4096, 11008)}
        Ys = {N: torch.empty((M, N), dtype=torch.float16, device="cuda") for N in (4096, 11008, 32000)}

        # batch 1: each run of INT4 modules is one qnt_gemv_seq call with the data
        # dependencies of a decode layer (q, k, v read the previous layer's down
        # output; o reads attention over q, k, v; gate and up read o's; down reads
        # gate's and up's), the INT8 modules qnt_gemv calls between them (each
        # module its own y, as the sequence call requires)
        producer = {0: -1, 1: -1, 2: -1, 3: 2, 4: 3, 5: 3, 6: 5}   # module in the layer -> producing module
        segments = []
        if M == 1:
            for i, (fmt, N, K, d, c, m) in enumerate(stack):
                y = torch.empty(N, dtype=torch.float16, device="cuda")
                l, j = divmod(i, 7)
                p = 7 * l + producer[j] if producer[j] >= 0 else 7 * l - 1   # global index of the producer
                if fmt == Q.QNT_INT4_ASYM and segments and segments[-1][0] == "seq" and \
                        len(segments[-1][1]) < Q.QNT_SEQ_MAX_STEPS:
                    start = segments[-1][2]
                    local = len(segments[-1][1])
                    segments[-1][1].append((d, c, m, Xs[K], y, local - (p - start) if p >= start else 0))
                elif fmt == Q.QNT_INT4_ASYM:
                    segments.append(("seq", [(d, c, m, Xs[K], y, 0)], i))
                else:
                    segments.append(("one", (d, c, m, Xs[K], y), i))
            segments = [(kind, (Q.seq_steps(v), torch.zeros(Q.qnt_gemv_seq_work_bytes(len(v)), dtype=torch.uint8,
                                                             device="cuda")) if kind == "seq" else v)
                        for kind, v, _ in segments]

        def run_stack(s, M=M, Xs=Xs, Ys=Ys, segments=segments):
            if M == 1:
                for kind, v in segments:
                    if kind == "seq":
                        Q.qnt_gemv_seq(v[0], 0, v[1], st, s)
                    else:
                        Q.qnt_gemv(*v, 0, st, s)
                return
            for fmt, N, K, d, c, m in stack:
                Q.qnt_gemm(d, c, m, Xs[K], Ys[N], M, 0, st, s)

        def run_head(s, M=M, Xs=Xs, Ys=Ys):
            d, c, m = head
            if M == 1:
                Q.qnt_gemv(d, c, m, Xs[4096], Ys[32000], 0, st, s)
            else:
                Q.qnt_gemm(d, c, m, Xs[4096], Ys[32000], M, 0, st, s)
        ms = _time_graph(torch, stream, run_stack, 3, 10)
        med = statistics.median(ms)
        out[f"selective_stack_b{M}"] = {
            "us_per_token_step": round(med * 1000.0, 1), "us_per_layer": round(med * 1000.0 / 32, 2),
            "p10_p90_ms": [round(pct(ms, 10), 4), round(pct(ms, 90), 4)],
            "GBps": round(stack_bytes[M] / (med * 1e-3) / 1e9, 1),
            "frac_hbm": round(stack_bytes[M] / (med * 1e-3) / 1e9 / hbm, 4),
            "how": ("224 modules (INT4 g128; INT8 per-channel down_proj in layers 0,1,30,31) in one CUDA graph: "
                    + (f"{sum(k == 'seq' for k, _ in segments)} qnt_gemv_seq calls with the decode-layer "
                       "dependencies for the INT4 runs, qnt_gemv for the INT8 modules" if M == 1 else
                       "224 qnt_gemm launches"))}
        hm = _time_graph(torch, stream, run_head, 3, 20)
        hmed = statistics.median(hm)
        hb = algo_bytes(6, 32000, 4096, M)
        out[f"lm_head_fp16_b{M}"] = {"us": round(hmed * 1000.0, 2), "GBps": round(hb / (hmed * 1e-3) / 1e9, 1),
                                     "frac_hbm": round(hb / (hmed * 1e-3) / 1e9 / hbm, 4)}
    assert int(st.item()) == 0
    del stack, head
    torch.cuda.empty_cache()
    return out


def run_kernel_only(name: str, fmt_name: str, M: int = 16, repeats: int = 5):
    """Small cases for profilers, each a few launches of one kernel:
      a layer shape (qkv, o, gate, up, down): one matrix of that shape, quantized
        once, then `repeats` qnt_gemv launches (batch 1, fp16 x);
      "layer": one decode layer (its five GEMVs, with the bench's waits) as
        `repeats` qnt_gemv_seq launches;
      "gemm": the Llama-70B gate/up matrix (K=8192, N=28672, INT4 g128) times M
        bf16 activation rows, `repeats` qnt_gemm launches;
      "quantize": qnt_quantize of the Llama-7B gate matrix (11008 x 4096 fp32);
      "int8_down": the INT8 per-channel down_proj (K=11008, N=4096), qnt_gemv;
      "fp16_lm_head": the FP16 lm_head (K=4096, N=32000), qnt_gemv."""
    import torch
    from dequant_gemv_rtn_b200 import qnt as Q
    from dequant_gemv_rtn_b200 import synth
    st = torch.zeros(1, dtype=torch.int32, device="cuda")

    def quantized(fmt, N, K, g, seed):
        d = Q.desc(fmt, N, K, g)
        W = synth.llama_like_device(N, K, seed=seed)
        codes = torch.empty(Q.qnt_codes_bytes(d), dtype=torch.uint8, device="cuda")
        meta = torch.empty(max(16, Q.qnt_meta_bytes(d)), dtype=torch.uint8, device="cuda")
        Q.qnt_quantize(d, W, codes, meta, st)
        return d, codes, meta

    shapes = []
    if name == "gemm":
        d, codes, meta = quantized(Q.QNT_INT4_ASYM, 28672, 8192, GROUP, 3)
        X = synth.activations_device(M, 8192, seed=5, dtype=torch.bfloat16)
        Y = torch.empty((M, 28672), dtype=torch.bfloat16, device="cuda")
        for _ in range(repeats):
            Q.qnt_gemm(d, codes, meta, X, Y, M, Q.QNT_BF16, st)
        shapes, outs = [[28672, 8192, M]], [Y]
    elif name == "quantize":
        d = Q.desc(Q.QNT_INT4_ASYM, INTER, HIDDEN, GROUP)
        W = synth.llama_like_device(INTER, HIDDEN, seed=3)
        codes = torch.empty(Q.qnt_codes_bytes(d), dtype=torch.uint8, device="cuda")
        meta = torch.empty(Q.qnt_meta_bytes(d), dtype=torch.uint8, device="cuda")
        for _ in range(repeats):
            Q.qnt_quantize(d, W, codes, meta, st)
        shapes, outs = [[INTER, HIDDEN]], []
    elif name in ("int8_down", "fp16_lm_head"):
        fmt, N, K = (Q.QNT_INT8_PERCHAN, HIDDEN, INTER) if name == "int8_down" else (Q.QNT_FP16, 32000, HIDDEN)
        d, codes, meta = quantized(fmt, N, K, K, 3)
        x = synth.activations_device(1, K, seed=5, dtype=torch.float16)
        y = torch.empty(N, dtype=torch.float16, device="cuda")
        for _ in range(repeats):
            Q.qnt_gemv(d, codes, meta, x, y, Q.QNT_F16, st)
        shapes, outs = [[N, K]], [y]
    else:
        fmt = Q.FORMATS[fmt_name]
        layer_wait = {"qkv": 0, "o": 1, "gate": 1, "up": 2, "down": 1}
        mats = []
        for i, (n, N, K) in enumerate(SHAPES):
            if name not in ("layer", n):
                continue
            d, codes, meta = quantized(fmt, N, K, GROUP, 3 + i)
            x = synth.activations_device(1, K, seed=5, dtype=torch.float16)
            y = torch.empty(N, dtype=torch.float16, device="cuda")
            mats.append((n, d, codes, meta, x, y))
        if name == "layer":
            steps = Q.seq_steps([(d, c, m, x, y, layer_wait[n]) for n, d, c, m, x, y in mats])
            work = torch.zeros(Q.qnt_gemv_seq_work_bytes(len(steps)), dtype=torch.uint8, device="cuda")
            for _ in range(repeats):
                Q.qnt_gemv_seq(steps, Q.QNT_F16, work, st)
        else:
            _, d, codes, meta, x, y = mats[0]
            for _ in range(repeats):
                Q.qnt_gemv(d, codes, meta, x, y, Q.QNT_F16, st)
        shapes, outs = [[d.N, d.K] for _, d, *_ in mats], [m[5] for m in mats]
    torch.cuda.synchronize()
    assert int(st.item()) == 0, f"device status {int(st.item())}"
    print(json.dumps({"kernel_only": name, "fmt": fmt_name, "launches": repeats, "shapes": shapes,
                      "y_finite": all(bool(torch.isfinite(o.float()).all()) for o in outs)}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--kernel-only", default=None,
                    choices=[n for n, _, _ in SHAPES] + ["layer", "gemm", "quantize", "int8_down", "fp16_lm_head"],
                    help="profiling case: a few launches of one kernel (see run_kernel_only)")
    ap.add_argument("--fmt", default="int4", help="format for --kernel-only with a layer shape")
    ap.add_argument("--m", type=int, default=16, help="activation rows for --kernel-only gemm")
    ap.add_argument("--repeats", type=int, default=5, help="launches for --kernel-only")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--no-extras", action="store_true", help="skip the other workloads")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.kernel_only:
        run_kernel_only(args.kernel_only, args.fmt, args.m, args.repeats)
        return
    world, rank, local = dist_setup(args.gpus)
    if args.impl == "reference":
        r = run_reference(args, world, rank, local)
        if r is not None:
            print(json.dumps(r), flush=True)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    import torch
    result, _ = run_ours(args, world, rank, local)
    if world == 1 and not args.no_extras:
        del _
        torch.cuda.empty_cache()
        result["extra_configs"] = run_extra_configs(args)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(torch, args.cpu_budget)
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
