#!/usr/bin/env python
"""Latent-MoE block forward (Muse Spark Open shapes) on B200: tokens/s and roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload prefill|decode|prefill_zipf|mid|tiny] [--no-side]

One step = one forward pass of the whole block (router, top-k, permutation, pooler,
gather, gate/up + SwiGLU, down + sum of squares, per-expert norm + combine, unpooler)
over one batch of synthetic tokens already resident in HBM, through the C ABI.
Default workload: the full-width prefill layer (T=8192, D=8192, L=4096, I=4096,
E=256, top-8, bf16); the decode layer (T=64) and the Zipf-skewed prefill are timed
beside it and reported as sub-objects. Multi-GPU: one process per GPU, every rank a
replica with its own tokens (weak scaling, no data-path collective), time = max over
ranks of the CUDA-event time.

Timing: W untimed warm-up steps, then K steps between CUDA events on the launching
stream, with a barrier and a device synchronisation on both sides. Every step streams
the expert weights (25.8 GB >> 126 MB L2), so inputs are larger than L2 and no flush is
needed. Per-kernel durations come from events the library records between its launches.
The side line "prefill_sublayer" runs the same layer inside its feed-forward sublayer
(pre-norm, block, post-norm, residual gate). Decode workloads are also timed as replays
of one CUDA graph of the forward
("graph_replay"), which takes the host's per-launch work out of the step.
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import json
import math
import os
import platform
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        try:
            d = json.load(open(p))
            if all(k in d for k in PEAKS_FALLBACK):
                return {k: float(d[k]) for k in PEAKS_FALLBACK}, "measured"
        except (ValueError, TypeError):
            pass
    return dict(PEAKS_FALLBACK), "fallback"


# ------------------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""
    Q = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = f"GPU-{torch.cuda.get_device_properties(device_index).uuid}"
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-lms", "100", "-i", self.dev], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self, t0: float, t1: float):
        rows = []
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((ts, float(f[1]), float(f[2]), f[5:9]))
            except ValueError:
                continue
        inside = [r for r in rows if t0 - 0.05 <= r[0] <= t1 + 0.05] or rows
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in inside for n, v in zip(names, r[3]) if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[1] for r in inside), "sm_max_mhz": max(r[2] for r in inside),
                "reasons": reasons, "samples": len(inside)}


# ------------------------------------------------------------------------------ accounting
def stage_work(w: W.Workload, n_touched: int):
    """Algorithmic FLOPs and bytes of each launch (only the k selected experts, only the
    distinct experts the routing touched; intermediates counted where a kernel's job is
    to move them)."""
    T, D, L, I, E, k = w.T, w.D, w.L, w.I, w.E, w.k
    a = 2 if w.dtype == "bf16" else 4
    ab = 0.5625 if w.experts == "nvfp4" else a      # bytes per expert weight
    aa = 0.5625 if w.act == "nvfp4" else a          # bytes per activation value the expert GEMMs read
    A = T * k
    return {
        "router": (2 * T * E * D, T * D * a + E * D * a + T * E * 4),
        "topk": (0, T * E * 4 + A * 8),
        "expert_hist": (0, A * 4),
        "tiles": (0, E * 8),
        "assign_rows": (0, A * 8),
        "pooler": (2 * T * L * D, T * D * a + L * D * a + T * L * a),
        "gather": (0, T * L * a + A * L * a),
        # W4A4: the GEMMs read their activation operands as codes (0.5625 B per value)
        "gate_up_swiglu": (2 * A * L * 2 * I, n_touched * 2 * I * L * ab + A * L * aa + A * I * a),
        "down_sumsq": (2 * A * I * L, n_touched * L * I * ab + A * I * aa + A * L * a + A * (L // 32) * 4),
        "norm_combine": (0, A * L * a + A * (L // 32) * 4 + T * L * a + n_touched * L * a),
        "unpooler": (2 * T * D * L, T * L * a + D * L * a + T * D * a),
        # optional steps: pre-expert norm on z; the feed-forward sublayer's pre-norm on x
        # and post-norm + residual gate (out, x, partial sums, gains, gate parameters)
        "pre_expert_norm": (0, 2 * T * L * a + L * a),
        "ffn_pre_norm": (0, 2 * T * D * a + D * a),
        "ffn_post_norm_gate": (0, 3 * T * D * a + T * (D // 32) * 4 + D * (a + 4)),
        # W4A4: latent rows quantised once per token (0.5625 B per value out), then gathered;
        # h quantised
        "quant_z": (0, T * L * a + T * L * 0.5625),
        "gather_codes": (0, T * L * 0.5625 + A * L * 0.5625),
        "quant_h": (0, A * I * a + A * I * 0.5625),
    }


def step_work(w: W.Workload, n_touched: int):
    """(FLOPs, bytes, the FLOPs that run on the FP4 tensor path) of one step."""
    T, D, L, I, E, k = w.T, w.D, w.L, w.I, w.E, w.k
    a = 2 if w.dtype == "bf16" else 4
    ab = 0.5625 if w.experts == "nvfp4" else a
    flops = 2 * T * (E * D + L * D + k * 3 * L * I + D * L)
    byts = 2 * T * D * a + (E * D + 2 * L * D) * a + n_touched * (3 * L * I * ab + L * a)
    fp4_flops = 2 * T * k * 3 * L * I if w.act == "nvfp4" else 0
    return flops, byts, fp4_flops


# ------------------------------------------------------------------------------ our arm
def rank_tokens(w: W.Workload, rank: int, dev) -> torch.Tensor:
    """Rank r's batch: tokens [rT, (r+1)T) of the workload's one seeded token stream, so N
    replicas together process N*T distinct tokens (weak scaling, no data-path exchange)."""
    x = torch.empty((w.T, w.D), dtype=W.TORCH_DTYPE[w.dtype], device=dev)
    return W.fill(x, w.seed, W.TID["x"], 1.0, start=rank * w.T * w.D)


def job_tokens_per_s(world: int, T: int, steps: int, ms_max: float) -> float:
    """Whole-job throughput: tokens of all ranks over the slowest rank's time."""
    return world * T * steps / (ms_max * 1e-3)


def make_rank_inputs(w: W.Workload, rank: int, dev):
    inp = W.make_inputs(w, dev, names=["W_router", "W_pool", "W_gate", "W_up", "W_down", "gamma", "W_unpool"])
    inp["x"] = rank_tokens(w, rank, dev)
    return inp


def time_graph(w: W.Workload, model, inp, out, idx, steps: int, warmup: int, world: int, dev):
    """The same forward captured once in a CUDA graph and replayed: CUDA-event time of
    `steps` replays (max over ranks), no host work between launches."""
    import latent_mixture_experts_moe_b200 as moe
    side = torch.cuda.Stream(device=dev)
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        model(inp["x"], out=out, topk_idx=idx)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        model(inp["x"], out=out, topk_idx=idx)
    for _ in range(warmup):
        graph.replay()
    torch.cuda.synchronize()
    barrier(world)
    stream = torch.cuda.current_stream()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        graph.replay()
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms = all_max(t0.elapsed_time(t1), world, dev)
    code, detail = moe.last_device_status(model.config(w.T, model.workspace))
    del graph
    if code != 0:
        raise RuntimeError(f"device status {code} detail {detail:#x} under graph replay")
    return {"value": job_tokens_per_s(world, w.T, steps, ms), "unit": "tokens/s", "ms_per_step": ms / steps,
            "steps": steps}


def run_ours(w: W.Workload, inp, steps: int, warmup: int, rank: int, world: int, peaks, peak_kind,
             sample_clocks: bool, e2e_steps: int, graph_steps: int = 0):
    import latent_mixture_experts_moe_b200 as moe
    dev = inp["x"].device
    weights = {k: v for k, v in inp.items() if k != "x"}
    modes = {"act_format": moe.ACT_NVFP4} if w.act == "nvfp4" else {}
    model = moe.LatentMoE(weights, T_max=w.T, k=w.k, eps=w.eps, **modes)
    out = torch.empty((w.T, w.D), dtype=inp["x"].dtype, device=dev)
    idx = torch.empty((w.T, w.k), dtype=torch.int32, device=dev)
    stage_names = moe.stages(model.config(w.T))
    nst = len(stage_names)
    stream = torch.cuda.current_stream()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nst + 1)] for _ in range(steps)]
    for row in ev:
        for e in row:
            e.record(stream)
    handles = [moe.event_handles(row) for row in ev]
    for _ in range(warmup):
        model(inp["x"], out=out, topk_idx=idx)
    torch.cuda.synchronize()
    code, detail = moe.last_device_status(model.config(w.T, model.workspace))
    if code != 0:
        raise RuntimeError(f"device status {code} detail {detail:#x}")
    clocks = ClockSampler(dev.index) if sample_clocks else None
    if clocks:
        clocks.start()
        time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    wall0 = time.time()
    t_start.record(stream)
    for s in range(steps):
        model(inp["x"], out=out, topk_idx=idx, stage_events=handles[s])
    t_end.record(stream)
    torch.cuda.synchronize()
    wall1 = time.time()
    barrier(world)
    if clocks:
        time.sleep(0.2)
        clocks.stop()
    ms = t_start.elapsed_time(t_end)
    ms_max = all_max(ms, world, dev)
    code, detail = moe.last_device_status(model.config(w.T, model.workspace))
    if code != 0:
        raise RuntimeError(f"device status {code} detail {detail:#x}")
    stage_ms = [sum(ev[s][i].elapsed_time(ev[s][i + 1]) for s in range(steps)) / steps for i in range(nst)]
    # each step's own duration (its first to its last library event): median, min, max
    per_step = sorted(ev[s][0].elapsed_time(ev[s][nst]) for s in range(steps))
    n_touched = int(torch.unique(idx).numel())
    work = stage_work(w, n_touched)
    dom = max(range(nst), key=lambda i: stage_ms[i])
    dname = stage_names[dom]
    fl, by = work[dname]
    t_dom = stage_ms[dom] * 1e-3
    # W4A4 expert GEMMs run on the FP4 tensor path: its peak is the measured bf16 peak times
    # the nominal dense FP4 / BF16 ratio (9 / 2.25 PFLOP/s)
    fp4_gemm = w.act == "nvfp4" and dname in ("gate_up_swiglu", "down_sumsq")
    ratio = 4.0 if fp4_gemm else 1.0
    t_tensor = fl / (ratio * peaks["bf16_tflops_sustained"] * 1e12)
    t_hbm = by / (peaks["hbm_gbs"] * 1e9)
    if t_tensor >= t_hbm:
        roof = {"bound": "tensor", "achieved": fl / t_dom / 1e12, "peak": ratio * peaks["bf16_tflops_sustained"],
                "unit": "TFLOP/s"}
        roof["frac_of_burst_peak"] = fl / t_dom / 1e12 / (ratio * peaks["bf16_tflops"])
    else:
        roof = {"bound": "hbm", "achieved": by / t_dom / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    # against the datasheet figures too: 8 TB/s HBM3e, 2.25 PFLOP/s dense bf16 (x 4 for FP4)
    roof["frac_of_spec"] = roof["achieved"] / (8000.0 if roof["bound"] == "hbm" else 2250.0 * ratio)
    roof["kernel"] = dname
    roof["peak_source"] = f"{peak_kind} ({'sustained' if roof['bound'] == 'tensor' else 'copy'})" + \
        (" x 4 (nominal FP4 / BF16 dense ratio)" if fp4_gemm and roof["bound"] == "tensor" else "")
    roof["algorithmic_flops"] = fl
    roof["algorithmic_bytes"] = by
    roof["traffic"] = measured_traffic(dname, w)
    sf, sb, sf4 = step_work(w, n_touched)
    t_step = ms_max / steps * 1e-3
    bf16_peak = peaks["bf16_tflops_sustained"] * 1e12
    step_roof = max((sf - sf4) / bf16_peak + sf4 / (4.0 * bf16_peak), sb / (peaks["hbm_gbs"] * 1e9))
    res = {
        "value": job_tokens_per_s(world, w.T, steps, ms_max),
        "ms_per_step": ms_max / steps,
        "stage_ms": {stage_names[i]: round(stage_ms[i], 4) for i in range(nst)},
        "step_ms": {"median": per_step[len(per_step) // 2], "min": per_step[0], "max": per_step[-1]},
        "roofline": roof,
        "step": {"tflops": sf / t_step / 1e12, "gbs": sb / t_step / 1e9, "roofline_ms": step_roof * 1e3,
                 "frac_of_step_roofline": step_roof / t_step, "distinct_experts": n_touched},
        "wall_s": wall1 - wall0,
        "gpu_launches": steps * moe.launch_count(model.config(w.T)),
    }
    if clocks:
        res["clocks"] = clocks.summary(wall0, wall1)
    if e2e_steps > 0:
        res["e2e"] = run_e2e(w, model, inp, e2e_steps, world, dev)
    if graph_steps > 0:
        res["graph"] = time_graph(w, model, inp, out, idx, graph_steps, warmup, world, dev)
    return res


def run_e2e(w, model, inp, steps, world, dev):
    """Same metric through the host-buffer entry point: each step copies its tokens from
    pinned host memory to the device and its output back (two pinned buffers each,
    alternating), with the library's batched call overlapping batch b's compute with
    batch b + 1's upload and batch b - 1's download. The timed region runs from an event
    before the first upload to an event after the last download."""
    import latent_mixture_experts_moe_b200 as moe
    dt = inp["x"].dtype
    x_hosts = [inp["x"].cpu().pin_memory() for _ in range(2)]
    out_hosts = [torch.empty((w.T, w.D), dtype=dt).pin_memory() for _ in range(2)]
    x_devs = [torch.empty_like(inp["x"]) for _ in range(2)]
    out_devs = [torch.empty((w.T, w.D), dtype=dt, device=dev) for _ in range(2)]
    cfg = model.config(w.T, model.workspace)
    wt = model.w
    args = (wt["W_router"], wt["W_pool"], wt["W_gate"], wt["W_up"], wt["W_down"], wt["gamma"], wt["W_unpool"])
    compute, up, down = torch.cuda.current_stream(), torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)

    def run(n):
        moe.forward_host_batches(cfg, [x_hosts[b % 2] for b in range(n)], [out_hosts[b % 2] for b in range(n)],
                                 x_devs, out_devs, *args, compute, up, down)
    run(3)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(up)
    run(steps)
    e.record(down)
    torch.cuda.synchronize()
    ms = all_max(s.elapsed_time(e), world, dev)
    nbytes = w.T * w.D * (2 if w.dtype == "bf16" else 4)
    return {"value": job_tokens_per_s(world, w.T, steps, ms), "unit": "tokens/s", "h2d_bytes_per_step": nbytes,
            "d2h_bytes_per_step": nbytes, "ms_per_step": ms / steps,
            "overlap": "batch b computes while b+1 uploads and b-1 downloads (two copy streams)"}


def measured_traffic(kernel: str, w: W.Workload):
    """DRAM bytes per launch from the committed ncu summary, if it matches this kernel
    source and workload; else None."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p))
        ent = d.get(f"{w.name}:{kernel}")
        if ent is None or ent.get("src_sha") != kernel_source_sha():
            return None
        return ent["bytes_per_launch"]
    except (ValueError, KeyError):
        return None


def kernel_source_sha():
    import hashlib
    h = hashlib.sha256()
    from latent_mixture_experts_moe_b200.build import KERNEL_SOURCES
    for f in KERNEL_SOURCES:
        h.update(open(os.path.join(ROOT, "latent_mixture_experts_moe_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


# ------------------------------------------------------------------------------ oracle arm
def oracle_sample(w: W.Workload, n_tokens: int, dev, widen: bool):
    """Host copies of what the oracle needs for tokens [0, n) of the workload: those x
    rows, the shared weights and the experts their routing touches (generated on `dev`
    with the shared seeded generator). widen=True converts them to float64 up front."""
    import oracle
    xr = torch.empty((n_tokens, w.D), dtype=W.TORCH_DTYPE[w.dtype], device=dev)
    W.fill(xr, w.seed, W.TID["x"], 1.0)
    shared = {n: W.make_tensor(w, n, dev).cpu() for n in ("W_router", "W_pool", "gamma", "W_unpool")}
    x = xr.cpu()
    bias = W.zipf_router_bias(w) if w.routing == "zipf" else None
    logits = oracle.router_logits(oracle.as_f64(x), oracle.as_f64(shared["W_router"]))
    idx, _, _ = oracle.route(logits, w.k, None if bias is None else oracle.as_f64(bias))
    experts = {}
    for e in np.unique(idx):
        experts[int(e)] = tuple(W.expert_slab(w, n, int(e), dev).cpu() for n in ("W_gate", "W_up", "W_down"))
    if widen:
        x = oracle.as_f64(x)
        shared = {n: oracle.as_f64(v) for n, v in shared.items()}
        experts = {e: tuple(oracle.as_f64(m) for m in v) for e, v in experts.items()}
        bias = None if bias is None else oracle.as_f64(bias)
    return x, shared, bias, experts


def time_oracle(w, x, shared, bias, experts):
    """Wall time of one oracle forward (as_f64 is a no-op on pre-widened arrays)."""
    import oracle
    f = oracle.as_f64
    t0 = time.perf_counter()
    oracle.latent_moe_forward(f(x), f(shared["W_router"]), f(shared["W_pool"]), lambda e: experts[e],
                              f(shared["gamma"]), f(shared["W_unpool"]), w.k, w.eps,
                              router_bias=None if bias is None else f(bias))
    return time.perf_counter() - t0


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or "unknown"


def cpu_baseline(w: W.Workload, dev, n_tokens: int):
    x, shared, bias, experts = oracle_sample(w, n_tokens, dev, widen=False)
    dt = time_oracle(w, x, shared, bias, experts)
    flops_per_token = 2 * (w.E * w.D + w.L * w.D + w.k * 3 * w.L * w.I + w.D * w.L)
    # the same oracle on one core (BLAS limited to one thread), one token, widening included
    one_core = None
    try:
        from threadpoolctl import threadpool_limits
        x1, shared1, bias1, experts1 = oracle_sample(w, 1, dev, widen=False)
        with threadpool_limits(limits=1):
            one_core = 1.0 / time_oracle(w, x1, shared1, bias1, experts1)
    except ImportError:
        pass
    return {"value": n_tokens / dt, "unit": "tokens/s", "cores": host_cores(), "kind": "oracle",
            "gflops_fp64": n_tokens * flops_per_token / dt / 1e9, "cpu_model": cpu_model(),
            "one_core_tokens_per_s": one_core,
            "sample": f"first {n_tokens} tokens of the {w.name} workload (T={w.T}) through the FP64 numpy "
                      f"oracle, widening bf16 weights to f64 included; {len(experts)} distinct experts; {dt:.1f} s"}


def run_reference(w: W.Workload, args, dev):
    """The FP64 oracle as the reference arm: every step runs the workload's first token
    through the whole block, on weights widened to float64 before timing."""
    x, shared, bias, experts = oracle_sample(w, 1, dev, widen=True)
    times = [time_oracle(w, x, shared, bias, experts) for _ in range(args.warmup + args.steps)][args.warmup:]
    total = sum(times)
    value = args.steps / total
    return {
        "metric": metric_name(), "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(w), "impl": "reference",
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": host_cores(), "kind": "oracle",
                         "sample": f"token 0 of the {w.name} workload per step, FP64 numpy oracle, "
                                   f"weights pre-widened to f64"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ------------------------------------------------------------------------------ plumbing
def metric_name():
    return "latent-MoE layer tokens/s on 1 B200 (T=8192 prefill, T=64 decode); % roofline"


def config_dict(w: W.Workload):
    return {"workload": f"{w.name}: latent-MoE layer T={w.T} D={w.D} L={w.L} I={w.I} E={w.E} top-{w.k} "
                        f"{w.dtype} {w.routing} routing",
            "T": w.T, "D": w.D, "L": w.L, "I": w.I, "E": w.E, "top_k": w.k, "routing": w.routing,
            "l2": "inputs larger than L2: each step streams the touched experts' weights (up to 25.8 GB)"}


_DIST = {"on": False}


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def all_max(v: float, world: int, dev) -> float:
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="prefill", choices=list(W.WORKLOADS))
    ap.add_argument("--no-side", action="store_true", help="skip the decode / skewed side workloads")
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle cpu_baseline")
    ap.add_argument("--no-nvfp4", action="store_true", help="skip the NVFP4-expert side workloads")
    ap.add_argument("--cpu-tokens", type=int, default=16)
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        # the FP64 oracle on the host cores: rank 0 alone, no process group; the seeded
        # inputs are generated on the GPU when there is one (same bytes either way)
        if rank == 0:
            dev = torch.device("cuda", local) if torch.cuda.is_available() else torch.device("cpu")
            print(json.dumps(run_reference(W.WORKLOADS[args.workload], args, dev)), flush=True)
        return
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=dev)
    w = W.WORKLOADS[args.workload]
    try:
        peaks, peak_kind = load_peaks()
        inp = make_rank_inputs(w, rank, dev)
        main_res = run_ours(w, inp, args.steps, args.warmup, rank, world, peaks, peak_kind, True,
                            e2e_steps=min(args.steps, 20),
                            graph_steps=args.steps if w.name.endswith("decode") else 0)
        side = {}
        if not args.no_side and w.name == "prefill":
            wd = W.WORKLOADS["decode"]
            inp_d = dict(inp, x=rank_tokens(wd, rank, dev))
            side["decode"] = run_ours(wd, inp_d, max(args.steps, 50), args.warmup, rank, world, peaks, peak_kind,
                                      False, e2e_steps=0, graph_steps=max(args.steps, 50))
            wz = W.WORKLOADS["prefill_zipf"]
            inp_z = dict(inp, router_bias=W.zipf_router_bias(wz).to(dev))
            side["prefill_zipf"] = run_ours(wz, inp_z, args.steps, args.warmup, rank, world, peaks, peak_kind,
                                            False, e2e_steps=0)
            # the whole feed-forward sublayer: pre-norm, the block, post-norm, residual gate
            inp_s = dict(inp, **W.sublayer_inputs(w, dev))
            side["prefill_sublayer"] = run_ours(w, inp_s, args.steps, args.warmup, rank, world, peaks, peak_kind,
                                                False, e2e_steps=0)
            if not args.no_nvfp4:
                # NVFP4 experts (quantised from the same bf16 weights): T=4096 and a T=64 decode
                wq = W.WORKLOADS["nvfp4"]
                q = W.make_inputs(wq, dev, names=["W_gate", "W_up", "W_down"])
                inp_q = dict({k: v for k, v in inp.items() if k not in ("W_gate", "W_up", "W_down")}, **q)
                inp_q["x"] = rank_tokens(wq, rank, dev)
                side["nvfp4"] = run_ours(wq, inp_q, args.steps, args.warmup, rank, world, peaks, peak_kind,
                                         False, e2e_steps=0)
                wqd = W.WORKLOADS["nvfp4_decode"]
                inp_qd = dict(inp_q, x=rank_tokens(wqd, rank, dev))
                side["nvfp4_decode"] = run_ours(wqd, inp_qd, max(args.steps, 50), args.warmup, rank, world, peaks,
                                                peak_kind, False, e2e_steps=0)
                # the same weights with NVFP4 activations (W4A4, tcgen05 kind::mxf4nvf4)
                side["nvfp4_w4a4"] = run_ours(W.WORKLOADS["nvfp4_w4a4"], inp_q, args.steps, args.warmup, rank, world,
                                              peaks, peak_kind, False, e2e_steps=0)
                side["nvfp4_w4a4_decode"] = run_ours(W.WORKLOADS["nvfp4_w4a4_decode"], inp_qd, max(args.steps, 50),
                                                     args.warmup, rank, world, peaks, peak_kind, False, e2e_steps=0,
                                                     graph_steps=max(args.steps, 50))
        if rank == 0:
            line = {
                "metric": metric_name(), "value": main_res["value"], "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": main_res["ms_per_step"],
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
                "data": "synthetic (seeded counter-based N(0,1) inputs, N(0,1/fan_in) weights)",
                "config": dict(config_dict(w), parallelism=f"replicas x{world}" if world > 1 else "single GPU"),
                "roofline": main_res["roofline"], "step_roofline": main_res["step"],
                "stage_ms": main_res["stage_ms"], "step_ms": main_res["step_ms"],
                "gpu_launches": main_res["gpu_launches"],
                "clocks": main_res.get("clocks"), "e2e": main_res.get("e2e"),
            }
            if "graph" in main_res:
                line["graph_replay"] = main_res["graph"]
            for name, r in side.items():
                line[name] = {"value": r["value"], "unit": "tokens/s", "ms_per_step": r["ms_per_step"],
                              "roofline": r["roofline"], "step_roofline": r["step"], "stage_ms": r["stage_ms"]}
                if "graph" in r:
                    line[name]["graph_replay"] = r["graph"]
            if world == 1 and not args.no_cpu:
                line["cpu_baseline"] = cpu_baseline(w, dev, args.cpu_tokens)
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
