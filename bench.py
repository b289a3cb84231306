#!/usr/bin/env python
"""Benchmark of the quantized MoE layer on B200: MoE-layer tokens/s and the roofline fraction.

One step = one full MoE layer forward (router + top-k, expert FFN, combine; plus permute for
prefill) over one batch of synthetic tokens, through the library's C ABI. Workloads (synthetic,
seeded; shapes from the pages' model: 512 experts, top-10, 48 layers, 8,192-token prefill
chunks, 1-4 token decode / MTP-verify passes):
  decode1   T=1,    H=2048, E=512, k=10, I=512, shared expert, Q2, Zipf(1.1) router bias   (default)
  decode4   T=4,    same
  prefill8k T=8192, uniform router, shared expert, Q2
  prefill2k_q3  T=2048, Q3, Zipf(1.2), no shared expert
Decode steps rotate over 48 distinct layer weight sets (24 GB, larger than L2) so the weights
come from HBM as in a real 48-layer decode; prefill steps rotate over 4 layers (503 MB each).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
Under torchrun each rank runs an independent replica (the layer shards by tokens with no
exchange); rank 0 prints one JSON line with the whole-job throughput (max time over ranks).
On one GPU the default run (decode1) also times decode4 (480 steps) and prefill8k (8 steps) and
reports them under "breakdown", so one line carries the metric at T = 1, 4 and 8192.
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
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

WORKLOADS = {
    "decode1": dict(shape="decode1", layers=48),
    "decode4": dict(shape="decode4", layers=48),
    "verify6": dict(shape="verify6", layers=48),
    "decode1_pruned256": dict(shape="decode1_pruned256", layers=48),
    "decode1_q4": dict(shape="decode1_q4", layers=48),
    "batch32": dict(shape="batch32", layers=48),
    "prefill8k": dict(shape="prefill8k", layers=4),
    "prefill2k_q3": dict(shape="prefill2k_q3", layers=4),
    # the 48-layer stack (RMSNorm before each router, residual stream, prefill-shaped layers with
    # a uniform router): one step = one token (decode, T=1) or one 8192-token chunk through all 48
    "stack_decode": dict(shape="stack", T=1, layers=48, stack=True),
    "stack_prefill": dict(shape="stack", T=8192, layers=48, stack=True),
}
METRIC = "MoE-layer tokens/s at T=1/4/8192; % of HBM or bf16 tensor-core roofline"
DEFAULT_STEPS = {"decode1": 4800, "decode4": 4800, "verify6": 4800, "decode1_pruned256": 4800, "decode1_q4": 4800,
                 "batch32": 960,
                 "prefill8k": 40, "prefill2k_q3": 60, "stack_decode": 256,
                 "stack_prefill": 4}
DEFAULT_WARMUP = {"decode1": 480, "decode4": 480, "verify6": 480, "decode1_pruned256": 480, "decode1_q4": 480,
                  "batch32": 96,
                  "prefill8k": 5, "prefill2k_q3": 5, "stack_decode": 16,
                  "stack_prefill": 3}


# extra workloads timed after the T=1 headline (steps, warm-up steps), and the keys kept for each
BREAKDOWN = {"decode4": (480, 48), "prefill8k": (8, 3)}
BREAKDOWN_KEYS = ("value", "unit", "steps", "warmup", "ms_per_step", "config", "roofline", "roofline_layer",
                  "kernels_us_per_step", "e2e", "gpu_launches", "clocks")


def workload_shape(name: str) -> synth.LayerShape:
    wl = WORKLOADS[name]
    if wl.get("stack"):
        st = synth.STACK
        return synth.LayerShape("stack", wl["T"], st["H"], st["E"], st["k"], st["I"], st["qtype"], st["shared"], None)
    return synth.WORKLOADS[wl["shape"]]


# DRAM bytes (read + write) per launch of the dominant kernels, from ncu captures of these kernel
# sources, valid only for the source and the launch shape they were taken on: the sources' sha256
# is checked at run time and the figure is dropped (traffic = null) once the source has changed,
# or for a workload whose launches differ from the captured one.
_DEC_SRC = ["quantized_expert_ffn_gemm_b200/csrc/decode_fused.cu", "quantized_expert_ffn_gemm_b200/csrc/common.cuh",
            "quantized_expert_ffn_gemm_b200/csrc/dequant.cuh", "quantized_expert_ffn_gemm_b200/csrc/gemv.cuh",
            "quantized_expert_ffn_gemm_b200/csrc/tc.cuh", "quantized_expert_ffn_gemm_b200/csrc/topk.cuh"]
_GEMM_SRC = ["quantized_expert_ffn_gemm_b200/csrc/gemm.cu", "quantized_expert_ffn_gemm_b200/csrc/tc.cuh",
             "quantized_expert_ffn_gemm_b200/csrc/dequant.cuh"]
_MID_SRC = ["quantized_expert_ffn_gemm_b200/csrc/mid.cu", "quantized_expert_ffn_gemm_b200/csrc/common.cuh",
            "quantized_expert_ffn_gemm_b200/csrc/dequant.cuh", "quantized_expert_ffn_gemm_b200/csrc/gemv.cuh"]
TRAFFIC = {
    # (kernel, workloads with the captured launch shape): (sources, sha256, DRAM bytes per launch)
    ("gemm_gate_up", ("prefill8k", "stack_prefill")):
        (_GEMM_SRC, "f08dad977b547aa9656127544c86817a1159fbae806114ced9b63f365c76169e", 862530560),
    ("decode_fused", ("decode1",)):
        (_DEC_SRC, "493d5f0ca9c45b0e25764ae7b0e4fb985de1c87211ce742466b031b77ba67e27", 15141120),
    ("mid_expert", ("batch32",)):
        (_MID_SRC, "542734f9d4c124de70b242a349a1d31e01fefbd186012371cec854041c2998e2", 46964736),
}


def traffic_for(kernel: str, workload: str):
    import hashlib
    ent = next((v for (kn, wls), v in TRAFFIC.items() if kn == kernel and workload in wls), None)
    if ent is None:
        return None
    srcs, sha, nbytes = ent
    h = hashlib.sha256()
    try:
        for src in srcs:
            with open(os.path.join(ROOT, src), "rb") as f:
                h.update(f.read())
    except OSError:
        return None
    return nbytes if h.hexdigest() == sha else None


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], tc=d["bf16_tflops"], tc_sus=d["bf16_tflops_sustained"], src="measured")
    return dict(hbm=6650.0, tc=1590.0, tc_sus=1400.0, src="fallback")


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.rows = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.Q,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                self.rows.append(parts)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in self.rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in self.rows for n, v in zip(names, r[5:9]) if v.strip().lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(self.rows)}


# ----------------------------------------------------------------------------- distributed
def dist_setup(backend: str | None = None):
    """One process per GPU: rank/world from the torchrun environment. NCCL on GPUs; gloo only
    where no GPU is present (the CPU tests of the multi-rank host logic)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if backend is None:
        backend = "nccl" if torch.cuda.is_available() else "gloo"
    if backend == "nccl":
        torch.cuda.set_device(local if world > 1 else 0)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    """The slowest rank's time: every rank contributes its own device-timed duration."""
    if world == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_throughput(tokens_per_step: int, steps: int, world: int, ms_max: float) -> float:
    """Tokens processed by all replicas / the slowest replica's time (weak scaling)."""
    return tokens_per_step * steps * world / (ms_max / 1e3)


def replica_x_stream(rank: int, i: int) -> int:
    """Input stream id of rank `rank`'s i-th token batch: replicas see distinct tokens."""
    return 1000 * rank + i


# ----------------------------------------------------------------------------- workload on device
def build_layers(shape: synth.LayerShape, n_layers: int, device="cuda"):
    """Per-layer device tensors: (Wr, bias, routed, shared); codes/scales drawn on the GPU."""
    layers = []
    for l in range(n_layers):
        Wr = synth.make_router(shape.seed, l, shape.E, shape.H).to(device)
        b = synth.zipf_bias(shape.seed, l, shape.E, shape.zipf_s).to(device) if shape.zipf_s else None
        rs = synth.make_expert_set(shape.seed, l, synth.SET_ROUTED, shape.qtype, shape.E, shape.H, shape.I, device)
        ss = (synth.make_expert_set(shape.seed, l, synth.SET_SHARED, shape.qtype, 1, shape.H, shape.I, device)
              if shape.shared else None)
        layers.append((Wr, b, rs, ss))
    return layers


def expert_bytes(shape: synth.LayerShape):
    """Packed bytes of one expert: (gate+up, down)."""
    per_w = {synth.Q2: 0.25, synth.Q3: 0.375, synth.Q4: 0.5}[shape.qtype] + 2.0 / 32  # codes + fp16 scale
    gu = 2 * shape.I * shape.H * per_w
    dn = shape.H * shape.I * per_w
    return gu, dn


def same_weights(a: synth.LayerShape, b: synth.LayerShape) -> bool:
    """Two workloads draw the same layer weights (they differ at most in T)."""
    return (a.H, a.E, a.k, a.I, a.qtype, a.shared, a.zipf_s, a.seed) == (b.H, b.E, b.k, b.I, b.qtype, b.shared,
                                                                         b.zipf_s, b.seed)


def run_ours(args, world, rank, local, workload=None, steps=None, warmup=None, layers=None):
    """Time `workload` (default: args.workload) for `steps` steps after `warmup` warm-up steps
    (default: args.steps / args.warmup); `layers` reuses another workload's device weights."""
    import quantized_expert_ffn_gemm_b200 as moe
    workload = workload or args.workload
    wl = WORKLOADS[workload]
    shape = workload_shape(workload)
    is_stack = bool(wl.get("stack"))
    T, H, E, k, I = shape.T, shape.H, shape.E, shape.k, shape.I
    n_layers = (args.layers if workload == args.workload else None) or wl["layers"]
    dev = torch.device("cuda", torch.cuda.current_device())
    if layers is None or len(layers) < n_layers:
        layers = build_layers(shape, n_layers)
    layers = layers[:n_layers]
    K = args.steps if steps is None else steps
    W = args.warmup if warmup is None else warmup
    ws = moe.Workspace.for_layer(H, E, k, I, shape.shared, T)
    y = torch.empty(T, H, dtype=torch.float32, device=dev)
    if is_stack:
        # independent seeded residual-stream inputs, one per step (tokens do not feed each other)
        n_x = min(K, 256) if T <= 8 else 2
        xs = [synth.make_residual(shape.seed, T, H, stream=replica_x_stream(rank, i)).to(dev) for i in range(n_x)]
        stack = moe.Stack([l[0] for l in layers], None, [l[2] for l in layers],
                          [l[3] for l in layers] if shape.shared else None, k)

        def step(i, x=None, idx_out=None):
            moe.stack_forward(xs[i % n_x] if x is None else x, stack, ws, eps=synth.STACK["eps"], r_out=y)

        def step_host(i, x_host, y_host):  # one C call: the copies and the stack
            moe.stack_forward_host(x_host, stack, ws, eps=synth.STACK["eps"], r_out_host=y_host)
    else:
        n_x = 64 if T <= 8 else 2
        xs = [synth.make_x(shape.seed, T, H, stream=replica_x_stream(rank, i)).to(dev) for i in range(n_x)]
        handles = [moe.LayerHandle(Wr, b, rs, ss, k, ws) for (Wr, b, rs, ss) in layers]

        path = {"auto": moe.PATH_AUTO, "gemm": moe.PATH_GEMM, "gemv": moe.PATH_GEMV, "mmq": moe.PATH_MMQ,
                "mid": moe.PATH_MID}[args.path]

        def step(i, x=None, idx_out=None):
            handles[i % n_layers].forward(xs[i % n_x] if x is None else x, y, idx_out=idx_out, path=path)

        def step_host(i, x_host, y_host):  # one C call: the copies and the layer
            handles[i % n_layers].forward_host(x_host, y_host, path=path)

    for i in range(W):
        step(i)
    torch.cuda.synchronize()
    assert moe.read_device_error(ws) == 0

    # ---------------- CUDA graphs: G consecutive steps per graph (one pass over the rotated layers;
    # a stack step already walks all layers, so its graphs hold 16 decode steps or one prefill chunk)
    if is_stack:
        G = min(16, K) if T <= 8 else 1
    else:
        G = n_layers if T <= 8 else min(n_layers, K)
    graphs = {}

    def graph_for(n, first):
        key = (n, first)
        if key not in graphs:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for j in range(n):
                    step(first + j)
            graphs[key] = g
        return graphs[key]

    if is_stack and T <= 8:  # every step of the pass its own token
        plan = [(G, j * G) for j in range(K // G)] + ([(K % G, (K // G) * G)] if K % G else [])
    else:
        plan = [(G, 0)] * (K // G) + ([(K % G, 0)] if K % G else [])
    for (n, f) in set(plan):
        graph_for(n, f).replay()
    torch.cuda.synchronize()

    # ---------------- timed region (device time, CUDA events on the launching stream)
    # The clock samples (nvidia-smi, 100 ms apart) span continuous replay of the same graphs: ~0.3 s
    # of it before the timed region and ~0.2 s after, so they see the load the timed steps run under
    # even when the timed region itself is shorter than one sampling interval.
    def soak(seconds):
        t_end = time.perf_counter() + seconds
        while time.perf_counter() < t_end:
            for (n, f) in plan:
                graphs[(n, f)].replay()
            torch.cuda.synchronize()

    clocks = ClockSampler(local)
    clocks.start()
    soak(0.3)
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for (n, f) in plan:
        graphs[(n, f)].replay()
    e1.record()
    torch.cuda.synchronize()
    barrier(world)
    ms = e0.elapsed_time(e1)
    soak(0.2)
    clk = clocks.stop()
    if clk is not None:
        clk["sampled"] = "continuous replay of the timed graphs, ~0.3 s before and ~0.2 s after the timed region"
    ms_max = max_over_ranks(ms, world)
    value = whole_job_throughput(T, K, world, ms_max)
    assert moe.read_device_error(ws) == 0

    # ---------------- per-kernel device time: blocks of G steps queued behind a sleep kernel so that
    # the event pair around each kernel brackets device execution, not host launch latency
    nblk = max(1, min(10 if T <= 8 else 3, K // G))
    if is_stack:
        nblk = 1
    idx_bufs = [torch.empty(T, k, dtype=torch.int32, device=dev) for _ in range(G)] if (T <= 128 and not is_stack) else None
    units_total = 0
    moe.timing_enable(True)
    for bi in range(nblk):
        torch.cuda._sleep(int(8e6))
        for j in range(G):
            step(j, idx_out=None if idx_bufs is None else idx_bufs[j])
        torch.cuda.synchronize()
        if idx_bufs is not None:
            units_total += sum(len(torch.unique(t)) + (1 if shape.shared else 0) for t in idx_bufs)
        elif T == 1:  # one token: its k experts are distinct
            units_total += G * (k + (1 if shape.shared else 0))
    moe.timing_enable(False)
    kt = moe.timing_read()
    Kt = nblk * G
    launches_per_step = sum(n for (_, n) in kt.values()) / Kt
    lps = n_layers if is_stack else 1  # layer passes per step
    Ktl = Kt * lps
    pk = peaks()

    if T <= 8 or "mid_expert" in kt:
        # decode: HBM bound. With the fused kernel the whole layer is one launch and its algorithmic
        # bytes are the distinct active experts + the fp32 router + x + y; with the separate kernels
        # the dominant one is the gate/up dequant-GEMV; on the mid-batch path the expert kernel
        # (every distinct expert's gate/up/down bytes, its partial rows written).
        # `achieved` counts the distinct active experts' packed bytes only (the benchmark spec's metric:
        # "% of HBM on active-expert bytes"); the all-bytes figure adds the fp32 router, x and y.
        gu_b, dn_b = expert_bytes(shape)
        units_avg = units_total / Kt
        if "decode_fused" in kt:
            dom = "decode_fused"
            algo = units_avg * (gu_b + dn_b)
            algo_all = algo + E * H * 4 + T * H * 2 + T * H * 4
        elif "mid_expert" in kt:
            dom = "mid_expert"
            algo = units_avg * (gu_b + dn_b)
            algo_all = algo + T * H * 2 + (I // 128) * (T * k + (T if shape.shared else 0)) * H * 4
        else:
            dom = "dec_gate_up"
            algo = units_avg * gu_b
            algo_all = algo + T * H * 2 + units_avg * T * I * 2
        d_ms, d_n = kt[dom]
        launch_us = d_ms / d_n * 1e3
        timing = "events around each launch (blocks queued behind a sleep kernel)"
        if set(kt) == {dom}:
            # the step is launches of this one kernel only: the timed region's events bracket them
            # back to back, without the per-launch event overhead (an upper bound: gaps included)
            launch_us = ms_max / K / (launches_per_step) * 1e3
            timing = "timed region (graph replay) / launches of the kernel in it; per-launch events gave %.2f us" % (
                d_ms / d_n * 1e3)
        achieved = algo / (launch_us / 1e6) / 1e9
        ach_all = algo_all / (launch_us / 1e6) / 1e9
        roof = {"kernel": dom, "bound": "hbm", "achieved": round(achieved, 1), "peak": pk["hbm"], "unit": "GB/s",
                "frac": round(achieved / pk["hbm"], 4), "traffic": traffic_for(dom, workload), "peak_source": pk["src"],
                "metric_bytes": "distinct active experts' packed bytes (north-star metric)",
                "algorithmic_bytes_per_launch": int(algo), "avg_launch_us": round(launch_us, 3),
                "all_bytes_per_launch": int(algo_all), "all_bytes_achieved": round(ach_all, 1),
                "all_bytes_frac": round(ach_all / pk["hbm"], 4),
                "distinct_experts_avg": round(units_avg, 2), "launch_timing": timing}
        layer_bytes = units_avg * (gu_b + dn_b) + E * H * 4 + T * H * 2 + T * H * 4
        layer_gbs = layer_bytes / (ms_max / K / lps / 1e3) / 1e9
        roof_layer = {"bound": "hbm", "bytes_per_step": int(layer_bytes), "achieved": round(layer_gbs, 1),
                      "frac": round(layer_gbs / pk["hbm"], 4), "distinct_experts_avg": round(units_avg, 2),
                      "note": "all bytes of a layer step (active experts + fp32 router + x + y) / step time"}
    else:
        rows = T * k + (T if shape.shared else 0)
        dom = "mmq_gate_up" if "mmq_gate_up" in kt else "gemm_gate_up"
        d_ms, d_n = kt[dom]
        flops = 2.0 * 2 * rows * H * I
        achieved = flops / (d_ms / d_n / 1e3) / 1e12
        # the burst peak unless the SM clock sagged under load (power cap): then the sustained one
        sm, smax = (clk or {}).get("sm_mhz"), (clk or {}).get("sm_max_mhz")
        capped = bool(sm and smax and sm < 0.95 * smax)
        peak_tc = pk["tc_sus"] if capped else pk["tc"]
        int8 = dom == "mmq_gate_up"
        if int8:  # int8 contraction: the bf16 figure times the nominal int8 / bf16 ratio (4.5 / 2.25 PF)
            peak_tc *= 2.0
        roof = {"kernel": dom, "bound": "tensor", "achieved": round(achieved, 1), "peak": peak_tc,
                "unit": "TFLOP/s", "frac": round(achieved / peak_tc, 4), "traffic": traffic_for(dom, workload),
                "peak_source": pk["src"] + (" sustained" if capped else " burst") +
                (" bf16 x 2 (int8 MMA, nominal ratio)" if int8 else
                 " bf16 (fp16 MMA runs at the bf16 rate)") + "; SM clock %s of %s MHz under load" % (sm, smax),
                "frac_of_other_peak": round(achieved / ((pk["tc"] if capped else pk["tc_sus"]) * (2.0 if int8 else 1.0)), 4),
                "algorithmic_flops_per_launch": flops, "avg_launch_us": round(d_ms / d_n * 1e3, 1)}
        layer_flops = 2.0 * 3 * rows * H * I + 2.0 * T * E * H
        tf = layer_flops / (ms_max / K / lps / 1e3) / 1e12
        roof_layer = {"bound": "tensor", "flops_per_step": layer_flops, "achieved": round(tf, 1),
                      "frac": round(tf / peak_tc, 4)}

    # ---------------- end to end through the public API with host buffers (pinned); the
    # host-to-device copy of each step's tokens and the read-back of y are inside the timed region
    Ke = min(K, 2000 if T <= 8 else 20)
    if is_stack:
        Ke = min(K, 64 if T <= 8 else 2)
    xh = [x.cpu().pin_memory() for x in xs[:8]]
    yh = torch.empty(T, H, dtype=torch.float32).pin_memory()
    step_host(0, xh[0], yh)  # warm-up of the host-buffer entry point
    torch.cuda.synchronize()
    barrier(world)
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record()
    for i in range(Ke):
        step_host(i, xh[i % len(xh)], yh)
    f1.record()
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(f0.elapsed_time(f1), world)
    e2e = {"value": round(whole_job_throughput(T, Ke, world, e2e_ms), 1), "unit": "tokens/s",
           "h2d_bytes_per_step": T * H * xs[0].element_size(),
           "d2h_bytes_per_step": T * H * 4, "steps": Ke,
           "note": "one C-ABI call per step from Python (%s: host-to-device copy of the step's tokens from "
                   "page-locked memory, the %s, device-to-host copy of the result), no graph" % (
               "moe_stack_forward_host" if is_stack else "moe_layer_forward_host", "stack" if is_stack else "layer")}
    del graphs

    out = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": round(ms_max / K, 6), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f16 (MMA operands; fp32 accumulate, router, y; weights Q2/Q3)", "data": "synthetic",
        "config": {"workload": f"{workload}: {'48-layer stack of MoE layers' if is_stack else 'MoE layer'} "
                               f"T={T}, H={H}, E={E}, top-{k}, I={I}, "
                               f"Q{shape.qtype}, shared={int(shape.shared)}, "
                               f"router bias={'Zipf(%s)' % shape.zipf_s if shape.zipf_s else 'none'}",
                   "T": T, "layers_rotated": n_layers, "graph_steps": G, "expert_path": args.path,
                   "l2": "inputs larger than L2: steps rotate over %d layer weight sets (%.1f GB)" % (
                       n_layers, n_layers * (layers[0][2].nbytes + (layers[0][3].nbytes if layers[0][3] else 0)
                                             + E * H * 4) / 1e9),
                   "parallelism": f"replicas x{world} (token-parallel, no collective)"},
        "roofline": roof, "roofline_layer": roof_layer,
        "kernels_us_per_step": {n: round(ms_ / Kt * 1e3, 3) for n, (ms_, _) in sorted(kt.items())},
        "ms_per_layer": round(ms_max / K / lps, 6),
        "e2e": e2e, "gpu_launches": int(round(launches_per_step * K)), "clocks": clk,
    }
    return out, shape, layers


def cpu_baseline(shape: synth.LayerShape, n_layers: int = 1, budget_s: float = 15.0):
    """The oracle, as it stands, on a bounded sample of the same workload on the host cores. For
    the 48-layer stack the sample is one layer's worth of tokens and the rate is divided by the
    layer count (extrapolated: every layer of the stack has the same shape and cost)."""
    import oracle
    L = synth.make_layer(shape)
    nthr = oracle.max_threads()
    t0 = time.time()
    oracle.layer_forward(L.x[:1], L.Wr, L.bias, shape.k, L.routed, L.shared, nthreads=1)
    one = max(time.time() - t0, 1e-3)                     # seconds per token on one core
    ntok = int(max(1, min(4 * nthr, budget_s / one * nthr)))
    xs = synth.make_x(shape.seed, ntok, shape.H, stream=777) if shape.T <= 8 else L.x[:ntok]
    t0 = time.time()
    oracle.layer_forward(xs, L.Wr, L.bias, shape.k, L.routed, L.shared, nthreads=nthr)
    dt = time.time() - t0
    value = ntok / dt / n_layers
    sample = (f"{ntok} independent tokens through the {shape.name} layer (layer 0 weights), "
              f"fp64 C oracle, one thread per token, {dt:.1f} s")
    if n_layers > 1:
        sample += f"; tokens/s divided by {n_layers} layers (extrapolated from one layer)"
    return {"value": round(value, 3), "unit": "tokens/s", "cores": min(nthr, ntok), "kind": "oracle",
            "sample": sample}


def run_reference(args, world, rank):
    """Reference arm: the CPU oracle on this arm's workload, timed on the host cores."""
    if rank != 0:
        return None
    import oracle
    wl = WORKLOADS[args.workload]
    shape = workload_shape(args.workload)
    lps = wl["layers"] if wl.get("stack") else 1
    L = synth.make_layer(shape)
    nthr = oracle.max_threads()
    T = shape.T
    # one step = the oracle on a bounded sample of the step's tokens (all of them when T <= 8);
    # for the stack, one layer of it, the rate divided by the layer count (extrapolated)
    sample_T = T if T <= 8 else min(T, 2 * nthr)
    mk = synth.make_residual if wl.get("stack") else synth.make_x
    xs = [mk(shape.seed, T, shape.H, stream=i)[:sample_T] for i in range(4)]
    if wl.get("stack"):
        xs = [oracle.rmsnorm_bf16(r, synth.STACK["eps"]) for r in xs]  # bf16 bits of the first layer's input
    warm, tw = 0, time.time()
    while warm < args.warmup and time.time() - tw < 60.0:  # the requested warm-up, within a minute
        oracle.layer_forward(xs[warm % 4], L.Wr, L.bias, shape.k, L.routed, L.shared, nthreads=nthr)
        warm += 1
    budget = 150.0
    t0 = time.time()
    done = 0
    for i in range(args.steps):
        oracle.layer_forward(xs[i % 4], L.Wr, L.bias, shape.k, L.routed, L.shared, nthreads=nthr)
        done += 1
        if time.time() - t0 > budget:
            break
    dt = time.time() - t0
    value = sample_T * done / dt / lps
    note = f"{done} steps x {sample_T} tokens of {shape.name}, fp64 C oracle"
    if lps > 1:
        note += f", one layer per step, rate divided by {lps} layers (extrapolated)"
    return {"metric": METRIC, "value": round(value, 3), "unit": "tokens/s", "n_gpus": world, "steps": done,
            "warmup": warm, "ms_per_step": round(dt / done * 1e3 * lps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": args.workload, "T": T, "sample_tokens_per_step": sample_T},
            "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": min(nthr, sample_T),
                             "kind": "oracle", "sample": note},
            "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_crossover(args):
    """Layer time at small batches through each expert path (the decode-to-prefill crossover):
    T tokens of the decode-shaped layer (H=2048, E=512, top-10, I=512, shared expert, Q2, Zipf(1.1)
    router bias), weights rotating over 8 layers, CUDA-event device time per call (calls issued one
    by one, and the same calls replayed from a CUDA graph), one JSON line per (T, path). Not a
    benchmark line of the contract: it informs the AUTO path's switch points."""
    import quantized_expert_ffn_gemm_b200 as moe
    torch.cuda.set_device(0)
    shape = synth.WORKLOADS["decode1"]
    H, E, k, I = shape.H, shape.E, shape.k, shape.I
    layers = build_layers(shape, 8)
    Tmax = 128
    ws = moe.Workspace.for_layer(H, E, k, I, True, Tmax)
    handles = [moe.LayerHandle(Wr, b, rs, ss, k, ws) for (Wr, b, rs, ss) in layers]
    xs = [synth.make_x(shape.seed, Tmax, H, stream=9000 + i).cuda() for i in range(8)]
    y = torch.empty(Tmax, H, dtype=torch.float32, device="cuda")
    paths = {"auto": moe.PATH_AUTO, "gemv": moe.PATH_GEMV, "gemm": moe.PATH_GEMM, "mid": moe.PATH_MID}
    for T in (1, 2, 4, 5, 6, 8, 12, 16, 24, 32, 48, 64, 96, 128):
        for name, path in paths.items():
            try:
                for i in range(8):
                    handles[i % 8].forward(xs[i % 8][:T], y[:T], path=path)
                torch.cuda.synchronize()
            except moe.MoeError as e:
                print(json.dumps({"T": T, "path": name, "unsupported": str(e)}), flush=True)
                continue
            n = 64
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for i in range(n):
                handles[i % 8].forward(xs[i % 8][:T], y[:T], path=path)
            e1.record()
            torch.cuda.synchronize()
            us = e0.elapsed_time(e1) / n * 1e3
            # the same calls replayed from a CUDA graph (eight layers per graph, eight replays)
            xg = [xs[i][:T].contiguous() for i in range(8)]
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for i in range(8):
                    handles[i].forward(xg[i], y[:T], path=path)
            g.replay()
            torch.cuda.synchronize()
            e0.record()
            for _ in range(8):
                g.replay()
            e1.record()
            torch.cuda.synchronize()
            us_graph = e0.elapsed_time(e1) / 64 * 1e3
            del g
            # per-kernel device time: the same calls queued behind a sleep kernel, events per launch
            nk = 16
            moe.timing_enable(True)
            torch.cuda._sleep(int(4e6))
            for i in range(nk):
                handles[i % 8].forward(xs[i % 8][:T], y[:T], path=path)
            torch.cuda.synchronize()
            moe.timing_enable(False)
            kt = {kn: round(ms_ / nk * 1e3, 2) for kn, (ms_, _) in sorted(moe.timing_read().items())}
            print(json.dumps({"T": T, "path": name, "us_per_layer": round(us, 2), "us_per_layer_graph": round(us_graph, 2),
                              "tokens_per_s": round(T / (us * 1e-6), 1), "kernels_us": kt}), flush=True)
    assert moe.read_device_error(ws) == 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--workload", default="decode1", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=None,
                    help="distinct layer weight sets to rotate over (default 48 for decode, 4 for prefill)")
    ap.add_argument("--path", default="auto", choices=["auto", "gemm", "gemv", "mmq", "mid"],
                    help="expert path of the layer workloads (mmq: int8 activations on tcgen05 kind::i8 for gate/up)")
    ap.add_argument("--no-breakdown", action="store_true",
                    help="time only --workload (by default a single-GPU run of the T=1 decode layer also times "
                         "the T=4 verify layer and the T=8192 prefill layer, reported under 'breakdown')")
    ap.add_argument("--crossover", action="store_true",
                    help="time the expert paths at T = 1..128 (one JSON line per T and path) and exit")
    args = ap.parse_args()
    if args.crossover:
        run_crossover(args)
        return
    if args.steps is None:
        args.steps = DEFAULT_STEPS[args.workload]
    if args.warmup is None:
        args.warmup = DEFAULT_WARMUP[args.workload]
    args.warmup = max(args.warmup, 3)

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        out = run_reference(args, world, rank)
        if out is not None:
            print(json.dumps(out), flush=True)
        return

    world, rank, local = dist_setup()
    try:
        out, shape, layers = run_ours(args, world, rank, local)
        if world == 1 and args.workload == "decode1" and not args.no_breakdown:
            # the metric is quoted at T = 1, 4 and 8192: the other two in the same run, each its own
            # timed region with fixed step counts (decode4 reuses the decode layers' weights)
            out["breakdown"] = {}
            for name, (K, W) in BREAKDOWN.items():
                o, _, _ = run_ours(args, world, rank, local, workload=name, steps=K, warmup=W,
                                   layers=layers if same_weights(shape, workload_shape(name)) else None)
                out["breakdown"][name] = {key: o[key] for key in BREAKDOWN_KEYS if key in o}
                torch.cuda.empty_cache()
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            wl = WORKLOADS[args.workload]
            out["cpu_baseline"] = cpu_baseline(shape, wl["layers"] if wl.get("stack") else 1)
        if rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
