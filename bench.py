#!/usr/bin/env python
"""Forward tokens/s of the TTT-Linear scan on B200 (1.3B-layer shape, 32k context).

One step = one ttt_linear_forward call over the whole workload
(B=2, H=32, T=32768, d=64, b=16, bf16 Q/K/V, fp32 state), inputs resident in
HBM.  tokens/s = B*T / step time (all H heads).  The inputs (1.35 GB per
step) are larger than the 126 MB L2, so no flush is needed between steps.

Multi-GPU (torchrun): every rank runs its own instance of the workload (the
(batch, head) scans are independent; no collective on the data path), so
scaling is weak and value = all ranks' tokens / max-over-ranks time.

--workload selects another of the synthetic workloads (the 125M-layer shape,
or the TTT-MLP layer, which reports against the bf16 tensor-core peak).
--impl reference times the float64 CPU oracle on a bounded sample of the
same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from test_sequence_layers_ttt_b200.inputs import WORKLOADS, make_inputs, select_heads  # noqa: E402

METRIC = "TTT forward tokens/sec on 1 B200 (1.3B-layer shape, 32k ctx); % of roofline"


def metric_name(w) -> str:
    if w.name == "linear_1p3b_32k":
        return METRIC
    if w.name == "decode_1p3b":
        return "TTT-Linear decode tokens/sec on 1 B200 (1.3B-layer shape, one token per sequence per step)"
    if w.name == "decode_mlp_8k":
        return "TTT-MLP decode tokens/sec on 1 B200 (TTT-MLP layer shape, one token per sequence per step)"
    shape = {"linear_125m_2k": "125M-layer shape, 2k ctx", "mlp_8k": "TTT-MLP layer, 8k ctx"}[w.name]
    return f"TTT forward tokens/sec on 1 B200 ({shape}); % of roofline"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
KEYS = ("Q", "K", "V", "eta", "W0", "b0", "gamma", "beta")
KEYS_MLP = ("Q", "K", "V", "eta", "W1_0", "b1_0", "W2_0", "b2_0", "gamma", "beta")


def algorithmic_bytes(w) -> int:
    """Bytes the scan must move: Q/K/V, eta, Z per head-token, the state read
    once and written once per (batch, head), gamma/beta once."""
    es = 2 if w.dtype == "bf16" else 4
    per_tok = 3 * w.d * es + 4 + 4 * w.d
    if w.kind == "mlp":
        state = 2 * (2 * w.d * w.hidden + w.hidden + w.d) * 4
    else:
        state = 2 * (w.d * w.d + w.d) * 4
    return w.head_tokens * per_tok + w.B * w.H * state + 2 * w.H * w.d * 4


def algorithmic_flops(w) -> int:
    """Per head-token.  Linear: 6 d^2 (X W, Q W, update) + 4*16*d (Q X^T, A G).
    MLP (hidden h): 7 products of 2 d h (two layers on K, two on Q, the hidden
    gradient, two updates) + 2*16*(2d + 2h) (the causal 16x16 terms)."""
    if w.kind == "mlp":
        return w.head_tokens * (7 * 2 * w.d * w.hidden + 2 * 16 * (2 * w.d + 2 * w.hidden))
    return w.head_tokens * (6 * w.d * w.d + 4 * 16 * w.d)


def load_peaks():
    """(HBM GB/s, dense bf16 TFLOP/s burst, 'measured' | 'fallback')."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            p = json.load(fh)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


KERNEL_SOURCES = {
    "ttt_linear_lag_kernel": ("ttt_linear_lag.cu", "ptx.cuh", "common.cuh", "tma_host.h", "ttt_internal.h"),
    "ttt_linear_umma_kernel": ("ttt_linear_umma.cu", "ptx.cuh", "tcgen05.cuh", "common.cuh", "tma_host.h",
                               "ttt_internal.h"),
    "ttt_linear_generic_kernel": ("ttt_linear_generic.cu", "common.cuh", "ttt_internal.h"),
    "ttt_mlp_tc_kernel": ("ttt_mlp_tc.cu", "ptx.cuh", "common.cuh", "ttt_internal.h"),
    "ttt_mlp_split_kernel": ("ttt_mlp_tc.cu", "ptx.cuh", "common.cuh", "ttt_internal.h"),
    "ttt_mlp_generic_kernel": ("ttt_mlp_generic.cu", "common.cuh", "ttt_internal.h"),
    "ttt_linear_decode_kernel": ("ttt_linear_decode.cu", "common.cuh", "ttt_internal.h"),
    "ttt_mlp_decode_kernel": ("ttt_mlp_decode.cu", "common.cuh", "ttt_internal.h"),
    "ttt_prologue_kernel": ("ttt_prologue.cu", "ptx.cuh", "tcgen05.cuh", "common.cuh", "tma_host.h",
                            "ttt_internal.h"),
    # the kernels of one ttt_linear_backward call: its own file, and the scan's checkpoint variant
    "ttt_linear_backward": ("ttt_linear_backward.cu", "ttt_linear_lag.cu", "ptx.cuh", "common.cuh", "tma_host.h",
                            "ttt_internal.h"),
}


def kernel_source_hash(kernel: str) -> str:
    """Hash of the source files a kernel is built from (its recorded counters
    stay valid while this does not change)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "test_sequence_layers_ttt_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, name), "rb") as fh:
            h.update(name.encode() + fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from
    the committed ncu summary, or None when the kernel sources changed since the
    counters were taken.  Lines: kernel workload source_hash bytes."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    with open(path) as fh:
        for line in fh:
            f = line.split("#")[0].split()
            if len(f) == 4 and f[0] == kernel and f[1] == workload:
                return int(f[3]) if f[2] == kernel_source_hash(kernel) else None
    return None


class ClockSampler:
    """Samples nvidia-smi SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in getattr(self, "lines", []):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=60))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def weak_scaling_value(w, world: int, ms_per_step: float) -> float:
    """Whole-job tokens/s: every rank processes its own B*T tokens (all H heads)
    per step; the step time is the max over ranks."""
    return w.B * w.T * world / (ms_per_step * 1e-3)


def dist_max(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def cpu_oracle_sample(w, inp, target_s: float):
    """Time the float64 oracle (all host cores) on whole (batch, head) scans of
    the workload, as many as fit in about target_s seconds; returns tokens/s in
    the workload's unit (B*T tokens cover all H heads)."""
    import oracle
    cores = os.cpu_count() or 1
    B, H = inp["Q"].shape[:2]
    pairs_all = [(b, h) for b in range(B) for h in range(H)]
    # calibrate on one scan
    def run(sel, threads):
        if w.kind == "mlp":
            oracle.ttt_mlp(*(sel[k] for k in KEYS_MLP), w.mini_batch, w.ln_eps, threads=threads)
        else:
            oracle.ttt_linear(*(sel[k] for k in KEYS), w.mini_batch, w.mode, w.ln_eps, threads=threads)

    sel = select_heads(inp, pairs_all[:1])
    t0 = time.perf_counter()
    run(sel, 1)
    one = time.perf_counter() - t0
    n = max(1, min(len(pairs_all), int(target_s / max(one, 1e-6) * min(cores, len(pairs_all)))))
    n = max(min(n, len(pairs_all)), 1)
    sel = select_heads(inp, pairs_all[:n])
    t0 = time.perf_counter()
    run(sel, cores)
    dt = time.perf_counter() - t0
    tokens = n * w.T / w.H
    used = min(cores, n)
    return {"value": tokens / dt, "unit": "tokens/s", "cores": used, "kind": "oracle",
            "sample": f"{n} of {w.B * w.H} (batch, head) scans at full T={w.T}, float64 primal oracle, "
                      f"{dt:.2f} s; tokens counted as scans*T/H"}


DECODE_WORKLOADS = ("decode_1p3b", "decode_mlp_8k")


def decode_state_bytes(w) -> int:
    """Algorithmic bytes of one decode step (one token for every (batch, head)
    stream): running state read and written, the mini-batch start state read
    and written, and the token's q, k, v, eta in and z out."""
    if w.kind == "mlp":
        state = 4 * (2 * w.d * w.hidden + w.hidden + w.d)
    else:
        state = 4 * (w.d * w.d + w.d)
    es = 2 if w.dtype == "bf16" else 4
    return w.B * w.H * (4 * state + 3 * w.d * es + 4 + w.d * 4)


def cpu_oracle_decode_sample(w, inp, target_s: float):
    """Time the float64 oracle's decode, one token per (batch, head) stream per
    step over the whole B x H batch, for about target_s seconds; tokens/s
    counts one token per sequence per step (B per step)."""
    import oracle
    cores = os.cpu_count() or 1
    if w.kind == "mlp":
        run, start = [inp[k] for k in ("W1_0", "b1_0", "W2_0", "b2_0")], [None] * 4
    else:
        W, b, W_mb, b_mb = inp["W0"], inp["b0"], None, None
    steps, t0 = 0, time.perf_counter()
    while True:
        i = steps % w.T
        sl = {k: inp[k][:, :, i:i + 1] for k in ("Q", "K", "V", "eta")}
        if w.kind == "mlp":
            out = oracle.ttt_mlp_decode(sl["Q"], sl["K"], sl["V"], sl["eta"], *run, *start, inp["gamma"],
                                        inp["beta"], w.mini_batch, i % w.mini_batch, w.ln_eps, threads=cores)
            run, start = list(out[1:5]), list(out[5:9])
        else:
            _, W, b, W_mb, b_mb = oracle.ttt_linear_decode(sl["Q"], sl["K"], sl["V"], sl["eta"], W, b, W_mb, b_mb,
                                                           inp["gamma"], inp["beta"], w.mini_batch,
                                                           i % w.mini_batch, w.mode, w.ln_eps, threads=cores)
        steps += 1
        dt = time.perf_counter() - t0
        if dt >= target_s:
            break
    return {"value": steps * w.B / dt, "unit": "tokens/s", "cores": min(cores, w.B * w.H), "kind": "oracle",
            "sample": f"{steps} single-token decode steps of all {w.B * w.H} (batch, head) streams, "
                      f"float64 primal oracle, {dt:.2f} s"}


def run_reference_prologue(args):
    p = PROLOGUES[args.workload]
    host = prologue_inputs(args.seed, p["B"], p["T"], p["H"], p["d"], p["d_model"])
    for _ in range(args.warmup):
        cpu_oracle_prologue_sample(p, host, 0.5)
    vals, r = [], None
    t_start = time.perf_counter()
    per_step = min(args.ref_seconds, 150.0 / max(args.steps, 1))
    for _ in range(args.steps):
        r = cpu_oracle_prologue_sample(p, host, per_step)
        vals.append(r["value"])
    elapsed = time.perf_counter() - t_start
    value = statistics.median(vals)
    print(json.dumps({
        "impl": "reference", "metric": prologue_metric(p),
        "value": value, "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * elapsed / max(args.steps, 1), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": p["name"], "B": p["B"], "T": p["T"], "H": p["H"], "d": p["d"],
                   "d_model": p["d_model"]},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": r["cores"], "kind": "oracle",
                         "sample": r["sample"]},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0}), flush=True)


def run_reference_backward(args):
    w = WORKLOADS[BACKWARD[args.workload]]
    host = make_inputs(w, args.seed)
    up = backward_upstream(w, args.seed)
    for _ in range(args.warmup):
        cpu_oracle_backward_sample(w, host, up, 0.5)
    vals, r = [], None
    t_start = time.perf_counter()
    per_step = min(args.ref_seconds, 150.0 / max(args.steps, 1))
    for _ in range(args.steps):
        r = cpu_oracle_backward_sample(w, host, up, per_step)
        vals.append(r["value"])
    elapsed = time.perf_counter() - t_start
    value = statistics.median(vals)
    print(json.dumps({
        "impl": "reference", "metric": f"TTT-Linear layer backward tokens/sec on 1 B200 ({w.name}); % of HBM roofline",
        "value": value, "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * elapsed / max(args.steps, 1), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(workload_config(w), workload=args.workload, forward_workload=w.name),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": r["cores"], "kind": "oracle",
                         "sample": r["sample"]},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0}), flush=True)


def run_reference(args, world, rank):
    if rank != 0:
        return
    if args.workload in PROLOGUES:
        return run_reference_prologue(args)
    if args.workload in BACKWARD:
        return run_reference_backward(args)
    w = WORKLOADS[args.workload]
    inp = make_inputs(w, args.seed)
    sample = cpu_oracle_decode_sample if args.workload in DECODE_WORKLOADS else cpu_oracle_sample
    for _ in range(args.warmup):
        sample(w, inp, 0.5)
    vals, samples = [], None
    t_start = time.perf_counter()
    per_step = min(args.ref_seconds, 150.0 / max(args.steps, 1))  # whole run within a few minutes
    for _ in range(args.steps):
        r = sample(w, inp, per_step)
        vals.append(r["value"])
        samples = r
    elapsed = time.perf_counter() - t_start
    value = statistics.median(vals)
    line = {
        "impl": "reference", "metric": metric_name(w), "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * elapsed / max(args.steps, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": samples["cores"],
                         "kind": "oracle", "sample": samples["sample"]},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def workload_config(w):
    if w.name in DECODE_WORKLOADS:
        mb_state = 4 * w.B * w.H * 2 * ((2 * w.d * w.hidden + w.hidden + w.d) if w.kind == "mlp" else (w.d * w.d + w.d))
        return {"workload": w.name, "B": w.B, "H": w.H, "d": w.d, "mini_batch": w.mini_batch,
                "qkv_dtype": w.dtype, "state_dtype": "f32",
                "inner_model": (f"x + LN(MLP {w.d}->{w.hidden}->{w.d}, GELU)" if w.kind == "mlp"
                                else "x + LN(xW + b)"),
                "step": "one token for each of the B x H streams; positions cycle through the mini-batch",
                "timed": "steps rounded up to whole mini-batch cycles",
                "l2": f"no flush: the {mb_state / 1e6:.1f} MB state stays in L2 between steps, as in a decode loop"}
    return {"workload": w.name, "B": w.B, "H": w.H, "T": w.T, "d": w.d, "mini_batch": w.mini_batch,
            "qkv_dtype": w.dtype, "state_dtype": "f32",
            "inner_model": (f"x + LN(MLP {w.d}->{w.hidden}->{w.d}, GELU)" if w.kind == "mlp"
                            else "x + LN(xW + b)"),
            "l2": "inputs (Q/K/V/eta) larger than the 126 MB L2; no flush"}


def graph_step_floor_ms(dev, steps_per_graph: int, replays: int) -> float:
    """Per-step time of a CUDA graph of `steps_per_graph` empty kernel nodes,
    replayed like the decode graphs: the launch-latency floor of one step."""
    x = torch.zeros(1, device=dev)
    s = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(s):
        for _ in range(3):
            x.add_(0.0)
    torch.cuda.synchronize(dev)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        for _ in range(steps_per_graph):
            x.add_(0.0)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(replays):
        graph.replay()
    b.record()
    torch.cuda.synchronize(dev)
    del graph
    return a.elapsed_time(b) / (replays * steps_per_graph)


def run_decode(args, world, rank, local):
    """Single-token decode steps through ttt_linear_decode (d = 64: the decode
    kernel with the state in registers) or ttt_mlp_decode (generic family)."""
    from test_sequence_layers_ttt_b200 import _binding as ttt

    w = WORKLOADS[args.workload]
    dev = torch.device("cuda", local)
    host = make_inputs(w, args.seed + rank)
    n_tok = w.T
    toks = [{k: host[k][:, :, i:i + 1].contiguous().to(dev) for k in ("Q", "K", "V", "eta")}
            for i in range(n_tok)]
    gam, bet = host["gamma"].to(dev), host["beta"].to(dev)
    Z = torch.empty((w.B, w.H, 1, w.d), dtype=torch.float32, device=dev)
    mb = w.mini_batch
    if w.kind == "mlp":
        mlp_run = [host[k].to(dev) for k in ("W1_0", "b1_0", "W2_0", "b2_0")]
        mlp_start = [x.clone() for x in mlp_run]

        def step(t, pos0, s):
            ttt.ttt_mlp_decode(t["Q"], t["K"], t["V"], t["eta"], *mlp_run, *mlp_start, gam, bet, pos0=pos0,
                               mini_batch=mb, ln_eps=w.ln_eps, Z=Z, stream=s)
    else:
        W, b = host["W0"].to(dev), host["b0"].to(dev)
        W_mb, b_mb = W.clone(), b.clone()

        def step(t, pos0, s):
            ttt.ttt_linear_decode(t["Q"], t["K"], t["V"], t["eta"], W, b, W_mb, b_mb, gam, bet, pos0=pos0,
                                  mini_batch=mb, ln_eps=w.ln_eps, Z=Z, stream=s)

    # Device rate: one mini-batch cycle of single-token steps (positions 0..b-1)
    # captured in a CUDA graph, replayed; a decode loop runs this way.
    stream = torch.cuda.current_stream(dev)
    for i in range(mb * max(1, -(-args.warmup // mb))):  # whole cycles: the graph starts at position 0
        step(toks[i % n_tok], i % mb, stream)
    torch.cuda.synchronize(dev)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        cap = torch.cuda.current_stream(dev)
        for i in range(mb):
            step(toks[i], i, cap)
    for _ in range(max(1, args.warmup // mb)):
        graph.replay()
    torch.cuda.synchronize(dev)
    dist_barrier(world)
    torch.cuda.synchronize(dev)
    replays = max(1, -(-args.steps // mb))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(replays)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        time.sleep(0.3)
        start.record(stream)
        for i in range(replays):
            ev[i][0].record(stream)
            graph.replay()
            ev[i][1].record(stream)
        end.record(stream)
        torch.cuda.synchronize(dev)
    dist_barrier(world)
    timed_steps = replays * mb
    total_ms = dist_max(start.elapsed_time(end), world)
    floor_ms = graph_step_floor_ms(dev, mb, replays)
    ms_per_step = total_ms / timed_steps
    kernel_ms = statistics.mean(a.elapsed_time(c) for a, c in ev) / mb
    value = w.B * world / (ms_per_step * 1e-3)
    del graph

    # end to end: each step's token from pinned host memory, z back to the host
    host_toks = [{k: v.pin_memory() for k, v in
                  ((k, host[k][:, :, i:i + 1].contiguous()) for k in ("Q", "K", "V", "eta"))}
                 for i in range(min(n_tok, args.steps))]
    z_host = torch.empty(Z.shape, dtype=torch.float32, pin_memory=True)
    h2d = sum(v.numel() * v.element_size() for v in host_toks[0].values())
    d2h = z_host.numel() * z_host.element_size()
    torch.cuda.synchronize(dev)
    dist_barrier(world)
    t0 = time.perf_counter()
    for i in range(args.steps):
        t = {k: v.to(dev, non_blocking=True) for k, v in host_toks[i % len(host_toks)].items()}
        step(t, i % mb, stream)
        z_host.copy_(Z, non_blocking=True)
        stream.synchronize()  # the step's z is on the host before the next token is known
    e2e_s = dist_max((time.perf_counter() - t0) / args.steps, world)

    cpu_base = None
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        cpu_base = cpu_oracle_decode_sample(w, host, min(args.ref_seconds, 5.0))
    if rank == 0:
        hbm, _, peak_kind = load_peaks()
        ab = decode_state_bytes(w)
        kname = ("ttt_mlp_decode_kernel" if w.kind == "mlp" else
                 "ttt_linear_decode_kernel" if w.d == 64 else "ttt_linear_generic_kernel")
        hbm_equiv = ab / (kernel_ms * 1e-3) / 1e9
        line = {
            "metric": metric_name(w), "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": timed_steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic", "config": workload_config(w),
            # The state stays in L2 between steps, so bytes over HBM bandwidth bounds nothing
            # here; a step is bound by latency.  The floor is the per-step time of the same
            # graph structure with each decode kernel replaced by an empty one.
            "roofline": {"bound": "latency", "achieved": 1e3 * kernel_ms, "peak": 1e3 * floor_ms,
                         "unit": "us per step", "frac": floor_ms / kernel_ms,
                         "traffic": recorded_traffic(kname, w.name),
                         "hbm_equivalent_gbs": hbm_equiv, "hbm_peak_gbs": hbm, "peak_kind": peak_kind,
                         "floor": "CUDA graph of one mini-batch cycle of empty kernel nodes, replayed",
                         "algorithmic_bytes_per_launch": ab, "kernel_ms": kernel_ms, "kernel": kname},
            "cpu_baseline": cpu_base,
            "e2e": {"value": w.B * world / e2e_s, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": timed_steps,
            "clocks": clk.summary(),
            "kernel_impl": "generic" if kname.endswith("generic_kernel") else "decode",
            "timing": "CUDA graph of one mini-batch cycle of steps, replayed; e2e: eager calls",
        }
        print(json.dumps(line), flush=True)


# The layer's prologue on the 1.3B-layer shape: x [2, 32768, 2048] bf16 against the
# Q/K/V and learning-rate weights of 32 heads of d = 64.
PROLOGUES = {
    "prologue_1p3b_32k": {"name": "prologue_1p3b_32k", "B": 2, "T": 32768, "H": 32, "d": 64, "d_model": 2048},
    # one 16k-token sequence (a quarter of the above, still larger than L2): the case that
    # multi-pass ncu captures of the prologue kernel run on
    "prologue_1p3b_16k": {"name": "prologue_1p3b_16k", "B": 1, "T": 16384, "H": 32, "d": 64, "d_model": 2048},
}


def prologue_metric(p) -> str:
    return (f"TTT prologue tokens/sec on 1 B200 (1.3B layer: d_model {p['d_model']}, {p['H']} heads of {p['d']}, "
            f"{p['T'] // 1024}k ctx); % of tensor roofline")


def prologue_inputs(seed: int, B: int, T: int, H: int, d: int, d_model: int):
    """Seeded synthetic prologue inputs: x ~ N(0, 1), every weight ~ N(0, 1/d_model)
    (bf16); b_lr ~ N(0, 1) fp32."""
    g = torch.Generator().manual_seed(seed)
    bf = lambda *shape, std: (torch.randn(shape, generator=g) * std).to(torch.bfloat16)
    x = bf(B, T, d_model, std=1.0)
    tq, tk, tv = (bf(H, d_model, d, std=d_model ** -0.5) for _ in range(3))
    tl = bf(H, d_model, std=d_model ** -0.5)
    bl = torch.randn(H, generator=g)
    return x, tq, tk, tv, tl, bl


def prologue_flops(p) -> int:
    """2 M d_model N with M = B T tokens and N = 3 H d + H output columns."""
    return 2 * p["B"] * p["T"] * p["d_model"] * (3 * p["H"] * p["d"] + p["H"])


def cpu_oracle_prologue_sample(p, host, target_s: float):
    """Time the float64 prologue oracle on the first tokens of batch 0, as many
    as fit in about target_s seconds; tokens/s."""
    import oracle.prologue as op
    x, tq, tk, tv, tl, bl = host
    n, dt = 16, 0.0
    while True:
        t0 = time.perf_counter()
        op.project(x[:1, :n], tq, tk, tv, tl, bl)
        dt = time.perf_counter() - t0
        if dt >= target_s / 4 or n >= p["T"]:
            break
        n = min(p["T"], n * 4)
    return {"value": n / dt, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{n} tokens of one sequence, all {p['H']} heads, float64 oracle (numpy einsum, one "
                      f"thread), {dt:.2f} s"}


def run_prologue(args, world, rank, local):
    """Forward tokens/s of ttt_prologue_forward on the 1.3B-layer shape."""
    from test_sequence_layers_ttt_b200 import _binding as ttt

    p = PROLOGUES[args.workload]
    dev = torch.device("cuda", local)
    host = prologue_inputs(args.seed + rank, p["B"], p["T"], p["H"], p["d"], p["d_model"])
    g = [t.to(dev) for t in host]
    B, T, H, d = p["B"], p["T"], p["H"], p["d"]
    Q, K, V = (torch.empty((B, H, T, d), dtype=torch.bfloat16, device=dev) for _ in range(3))
    eta = torch.empty((B, H, T), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(x):
        st = ttt.lib.ttt_prologue_forward(B, T, H, d, p["d_model"], 0, 1.0, 10000.0, 1, ttt._ptr(x),
                                          *(ttt._ptr(t) for t in g[1:]), ttt._ptr(Q), ttt._ptr(K), ttt._ptr(V),
                                          ttt._ptr(eta), ttt._stream_handle(dev, stream))
        ttt._check(st)

    for _ in range(args.warmup):
        step(g[0])
    torch.cuda.synchronize(dev)
    dist_barrier(world)
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        time.sleep(0.3)
        start.record(stream)
        for i in range(args.steps):
            ev[i][0].record(stream)
            step(g[0])
            ev[i][1].record(stream)
        end.record(stream)
        torch.cuda.synchronize(dev)
    dist_barrier(world)
    ms_per_step = dist_max(start.elapsed_time(end), world) / args.steps
    kernel_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    value = B * T * world / (ms_per_step * 1e-3)

    # end to end: x from pinned host memory, Q/K/V/eta back to pinned host memory
    x_host = host[0].pin_memory()
    outs_host = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in (Q, K, V, eta)]
    h2d = x_host.numel() * x_host.element_size()
    d2h = sum(t.numel() * t.element_size() for t in outs_host)
    x_dev = torch.empty_like(g[0])
    e2e_steps = max(3, min(args.steps, 10))
    torch.cuda.synchronize(dev)
    dist_barrier(world)
    t0 = time.perf_counter()
    for _ in range(e2e_steps):
        x_dev.copy_(x_host, non_blocking=True)
        step(x_dev)
        for o, t in zip(outs_host, (Q, K, V, eta)):
            o.copy_(t, non_blocking=True)
        stream.synchronize()
    e2e_s = dist_max((time.perf_counter() - t0) / e2e_steps, world)

    cpu_base = None
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        cpu_base = cpu_oracle_prologue_sample(p, host, min(args.ref_seconds, 10.0))
    if rank == 0:
        _, bf16_tf, peak_kind = load_peaks()
        af = prologue_flops(p)
        achieved = af / (kernel_ms * 1e-3) / 1e12
        line = {
            "metric": prologue_metric(p),
            "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": p["name"], "B": B, "T": T, "H": H, "d": d, "d_model": p["d_model"],
                       "outputs": "Q, K, V bf16 [B][H][T][d] (rotary on Q, K), eta fp32 [B][H][T]",
                       "l2": f"inputs (x {B * T * p['d_model'] * 2 / 1e6:.0f} MB) and outputs (Q/K/V "
                             f"{3 * B * T * H * d * 2 / 1e6:.0f} MB) larger than the 126 MB L2; no flush"},
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": bf16_tf, "unit": "TFLOP/s",
                         "frac": achieved / bf16_tf, "traffic": recorded_traffic("ttt_prologue_kernel", p["name"]),
                         "peak_kind": peak_kind, "algorithmic_flops_per_launch": af, "kernel_ms": kernel_ms,
                         "kernel": "ttt_prologue_kernel"},
            "cpu_baseline": cpu_base,
            "e2e": {"value": B * T * world / e2e_s, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": args.steps,
            "clocks": clk.summary(),
        }
        print(json.dumps(line), flush=True)


# The layer backward on a forward workload's shapes.
BACKWARD = {"backward_1p3b_32k": "linear_1p3b_32k", "backward_125m_2k": "linear_125m_2k"}


def backward_bytes(w) -> int:
    """Algorithmic bytes of one ttt_linear_backward call: Q, K, V, eta and dZ
    read and dQ, dK, dV, deta written once per head-token; W0, b0, dW_T, db_T
    read and dW0, db0 written once per (batch, head); and the start state of
    every mini-batch written once and read once (the method's checkpoints)."""
    es = 2 if w.dtype == "bf16" else 4
    per_tok = 3 * w.d * es + 4 + 4 * w.d + 3 * 4 * w.d + 4
    state = (w.d * w.d + w.d) * 4
    n_mb = -(-w.T // w.mini_batch)
    return w.head_tokens * per_tok + w.B * w.H * (3 * state + 2 * n_mb * state)


def backward_upstream(w, seed: int):
    g = torch.Generator().manual_seed(1000 + seed)
    return (torch.randn((w.B, w.H, w.T, w.d), generator=g), torch.randn((w.B, w.H, w.d, w.d), generator=g),
            torch.randn((w.B, w.H, w.d), generator=g))


def cpu_oracle_backward_sample(w, host, up, target_s: float):
    """Time the float64 backward oracle (torch autograd over the token loop) on
    the first tokens of one (batch, head) scan, as many as fit in about
    target_s seconds; tokens/s in the workload's unit (B*T tokens cover all H
    heads, so a single head's tokens count 1/H)."""
    from oracle import backward as ob
    sel = lambda t: t[:1, :1]
    n, dt = 16, 0.0
    while True:
        sl = {k: (sel(host[k])[:, :, :n] if k in ("Q", "K", "V", "eta") else
                  (host[k][:1] if k in ("gamma", "beta") else sel(host[k]))) for k in KEYS}
        t0 = time.perf_counter()
        ob.ttt_linear_backward(*(sl[k].double().numpy() for k in KEYS), sel(up[0])[:, :, :n].double().numpy(),
                               w.mini_batch, w.mode, w.ln_eps, sel(up[1]).double().numpy(),
                               sel(up[2]).double().numpy())
        dt = time.perf_counter() - t0
        if dt >= target_s / 4 or n >= w.T:
            break
        n = min(w.T, n * 4)
    return {"value": n / w.H / dt, "unit": "tokens/s", "cores": torch.get_num_threads(), "kind": "oracle",
            "sample": f"{n} tokens of one (batch, head) scan, float64 autograd oracle, {dt:.2f} s; "
                      f"tokens counted as head-tokens/H"}


def run_backward(args, world, rank, local):
    """Tokens/s of ttt_linear_backward (all three kernels of one call)."""
    from test_sequence_layers_ttt_b200 import _binding as ttt

    w = WORKLOADS[BACKWARD[args.workload]]
    dev = torch.device("cuda", local)
    host = make_inputs(w, args.seed + rank)
    up = backward_upstream(w, args.seed + rank)
    g = {k: v.to(dev) for k, v in host.items()}
    dZ, dW, db = (t.to(dev) for t in up)
    f32 = dict(dtype=torch.float32, device=dev)
    outs = [torch.empty((w.B, w.H, w.T, w.d), **f32) for _ in range(3)] + [
        torch.empty((w.B, w.H, w.T), **f32), torch.empty((w.B, w.H, w.d, w.d), **f32),
        torch.empty((w.B, w.H, w.d), **f32), torch.empty((w.H, w.d), **f32), torch.empty((w.H, w.d), **f32)]
    need = ttt.linear_backward_workspace_size(w.B, w.H, w.T, w.d, w.mini_batch)
    ws = torch.empty(need, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(src, dz, dw, dbb):
        st = ttt.lib.ttt_linear_backward(
            w.B, w.H, w.T, w.d, w.mini_batch, ttt._dtype_code(src["Q"]), ttt._mode_code("ln"), float(w.ln_eps),
            *(ttt._ptr(src[k]) for k in KEYS), ttt._ptr(dz), ttt._ptr(dw), ttt._ptr(dbb),
            *(ttt._ptr(o) for o in outs), ttt._ptr(ws), ctypes.c_size_t(need), ttt._stream_handle(dev, stream))
        ttt._check(st)

    for _ in range(args.warmup):
        step(g, dZ, dW, db)
    torch.cuda.synchronize(dev)
    dist_barrier(world)
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        time.sleep(0.3)
        start.record(stream)
        for i in range(args.steps):
            ev[i][0].record(stream)
            step(g, dZ, dW, db)
            ev[i][1].record(stream)
        end.record(stream)
        torch.cuda.synchronize(dev)
    dist_barrier(world)
    ms_per_step = dist_max(start.elapsed_time(end), world) / args.steps
    call_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    value = w.B * w.T * world / (ms_per_step * 1e-3)

    # end to end: every input from pinned host memory, every gradient back
    host_in = {k: v.pin_memory() for k, v in host.items()}
    up_in = [t.pin_memory() for t in up]
    outs_host = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in outs]
    h2d = sum(v.numel() * v.element_size() for v in host_in.values()) + sum(
        t.numel() * t.element_size() for t in up_in)
    d2h = sum(o.numel() * o.element_size() for o in outs_host)
    dev_in = {k: torch.empty_like(v) for k, v in g.items()}
    dev_up = [torch.empty_like(t) for t in (dZ, dW, db)]
    e2e_steps = max(3, min(args.steps, 10))
    torch.cuda.synchronize(dev)
    dist_barrier(world)
    t0 = time.perf_counter()
    for _ in range(e2e_steps):
        for k in KEYS:
            dev_in[k].copy_(host_in[k], non_blocking=True)
        for d_, h_ in zip(dev_up, up_in):
            d_.copy_(h_, non_blocking=True)
        step(dev_in, *dev_up)
        for oh, o in zip(outs_host, outs):
            oh.copy_(o, non_blocking=True)
        stream.synchronize()
    e2e_s = dist_max((time.perf_counter() - t0) / e2e_steps, world)

    cpu_base = None
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        cpu_base = cpu_oracle_backward_sample(w, host, up, min(args.ref_seconds, 10.0))
    if rank == 0:
        hbm, _, peak_kind = load_peaks()
        ab = backward_bytes(w)
        achieved = ab / (call_ms * 1e-3) / 1e9
        line = {
            "metric": f"TTT-Linear layer backward tokens/sec on 1 B200 ({w.name}); % of HBM roofline",
            "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic",
            "config": dict(workload_config(w), workload=args.workload, forward_workload=w.name,
                           workspace_bytes=need,
                           step="one ttt_linear_backward call: states, reverse sweep, dgamma/dbeta (3 kernels)"),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                         "traffic": recorded_traffic("ttt_linear_backward", args.workload),
                         "peak_kind": peak_kind, "algorithmic_bytes_per_launch": ab,
                         "kernel_ms": call_ms, "kernel": "ttt_linear_backward (3 kernels)"},
            "cpu_baseline": cpu_base,
            "e2e": {"value": w.B * w.T * world / e2e_s, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": 3 * args.steps,
            "clocks": clk.summary(),
        }
        print(json.dumps(line), flush=True)


def run_ours(args, world, rank, local):
    from test_sequence_layers_ttt_b200 import _binding as ttt

    if args.workload in PROLOGUES:
        return run_prologue(args, world, rank, local)
    if args.workload in BACKWARD:
        return run_backward(args, world, rank, local)
    w = WORKLOADS[args.workload]
    if w.name in DECODE_WORKLOADS:
        return run_decode(args, world, rank, local)
    dev = torch.device("cuda", local)
    host = make_inputs(w, args.seed + rank)
    g = {k: v.to(dev) for k, v in host.items()}
    Z = torch.empty((w.B, w.H, w.T, w.d), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    if w.kind == "mlp":
        keys = KEYS_MLP
        state = {n: torch.empty_like(g[n + "_0"]) for n in ("W1", "b1", "W2", "b2")}
        outs = [Z, *state.values()]

        def call(inputs, **kw):
            return ttt.ttt_mlp_forward(*(inputs[k] for k in keys), mini_batch=w.mini_batch,
                                       ln_eps=w.ln_eps, **kw)

        def step(st=stream):
            call(g, impl=args.kernel, Z=Z, W1_T=state["W1"], b1_T=state["b1"], W2_T=state["W2"],
                 b2_T=state["b2"], stream=st)
    else:
        keys = KEYS
        W_T = torch.empty_like(g["W0"])
        b_T = torch.empty_like(g["b0"])
        outs = [Z, W_T, b_T]

        def call(inputs, **kw):
            return ttt.ttt_linear_forward(*(inputs[k] for k in keys), mini_batch=w.mini_batch,
                                          ln_eps=w.ln_eps, **kw)

        def step(st=stream):
            call(g, impl=args.kernel, Z=Z, W_T=W_T, b_T=b_T, stream=st)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    # Device rate: one call captured in a CUDA graph and replayed, so that the host's
    # per-call work (argument checks, tensor-map encoding) does not leave the GPU idle
    # between short launches; the end-to-end leg below times the plain calls.
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step(torch.cuda.current_stream(dev))
    graph.replay()
    torch.cuda.synchronize(dev)
    dist_barrier(world)
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        time.sleep(0.3)  # let the sampler start
        start.record(stream)
        for i in range(args.steps):
            ev[i][0].record(stream)
            graph.replay()
            ev[i][1].record(stream)
        end.record(stream)
        torch.cuda.synchronize(dev)
    dist_barrier(world)
    del graph
    total_ms = start.elapsed_time(end)
    per_launch_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = dist_max(total_ms, world)
    ms_per_step = total_ms / args.steps
    kernel_ms = statistics.mean(per_launch_ms)
    tokens_per_step = w.B * w.T * world
    value = weak_scaling_value(w, world, ms_per_step)

    # end to end through the public API with pinned host buffers
    host_in = {k: v.pin_memory() for k, v in host.items() if v is not None}
    h2d = sum(v.numel() * v.element_size() for v in host_in.values())
    d2h = sum(o.numel() * o.element_size() for o in outs)
    call(host_in)
    torch.cuda.synchronize(dev)
    dist_barrier(world)
    e2e_steps = max(5, min(args.steps, 20))
    t0 = time.perf_counter()
    for _ in range(e2e_steps):
        call(host_in)  # returns after the device->host copies finish
    e2e_s = dist_max((time.perf_counter() - t0) / e2e_steps, world)
    e2e_value = tokens_per_step / e2e_s

    cpu_base = None
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        cpu_base = cpu_oracle_sample(w, host, args.ref_seconds)

    if rank == 0:
        hbm, bf16_tf, peak_kind = load_peaks()
        ab = algorithmic_bytes(w)
        af = algorithmic_flops(w)
        if w.kind == "mlp":
            family = args.kernel if args.kernel != "auto" else ttt.mlp_pick_impl(
                w.B, w.H, w.T, w.d, w.hidden, w.mini_batch, w.dtype)
            kname = {"tensorcore": "ttt_mlp_tc_kernel", "tensorcore_split": "ttt_mlp_split_kernel",
                     "generic": "ttt_mlp_generic_kernel"}[family]
            achieved, peak, bound, unit = af / (kernel_ms * 1e-3) / 1e12, bf16_tf, "tensor", "TFLOP/s"
        else:
            family = args.kernel if args.kernel != "auto" else ttt.linear_pick_impl(
                w.B, w.H, w.T, w.d, w.mini_batch, w.dtype, w.mode)
            kname = {"tensorcore": "ttt_linear_lag_kernel", "tcgen05": "ttt_linear_umma_kernel",
                     "generic": "ttt_linear_generic_kernel"}[family]
            achieved, peak, bound, unit = ab / (kernel_ms * 1e-3) / 1e9, hbm, "hbm", "GB/s"
        traffic = recorded_traffic(kname, w.name)
        line = {
            "metric": metric_name(w), "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic", "config": workload_config(w),
            "roofline": {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
                         "frac": achieved / peak, "traffic": traffic, "peak_kind": peak_kind,
                         "algorithmic_bytes_per_launch": ab, "algorithmic_flops_per_launch": af,
                         "kernel_ms": kernel_ms, "kernel": kname},
            "cpu_baseline": cpu_base,
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": args.steps,
            "clocks": clk.summary(),
            "kernel_impl": family,
            "timing": "one call captured in a CUDA graph, replayed once per step; e2e: plain calls",
            "tflops_achieved": af / (kernel_ms * 1e-3) / 1e12,
            "hbm_gbs_achieved": ab / (kernel_ms * 1e-3) / 1e9,
        }
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="linear_1p3b_32k",
                    choices=[k for k, v in WORKLOADS.items() if v.T >= 2048 or k in DECODE_WORKLOADS]
                    + [*PROLOGUES, *BACKWARD])
    ap.add_argument("--kernel", choices=["auto", "generic", "tensorcore", "tensorcore_split", "tcgen05"],
                    default="auto")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--ref-seconds", type=float, default=10.0,
                    help="CPU seconds of oracle work per reference sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # one process per GPU: start the ranks with torchrun on this node
        cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
               "--master-addr", "127.0.0.1", "--master-port", os.environ.get("MASTER_PORT", "29511"),
               os.path.abspath(__file__), *sys.argv[1:]]
        sys.exit(subprocess.call(cmd))
    world, rank, local = dist_setup()
    if args.gpus != world:
        raise SystemExit(f"--gpus {args.gpus} but {world} ranks were started")
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
