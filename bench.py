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


def at_full_clock(clk) -> bool:
    """True when the timed region ran at the GPU's maximum SM clock with no power-cap
    throttling sampled (median within 3% of max, sw_power_cap never active): the burst GEMM
    peak, measured at that clock, is then the tensor roofline. Otherwise the sustained peak
    (measured under the 1 kW power cap) is: clock counters read inside the expert GEMMs show
    that under the cap their SM clock falls to ~1.3 GHz even when 100 ms nvidia-smi samples
    mostly report the maximum."""
    if not clk or not clk.get("sm_mhz") or not clk.get("sm_max_mhz"):
        return False
    return clk["sm_mhz"] >= 0.97 * clk["sm_max_mhz"] and "sw_power_cap" not in clk.get("reasons", [])


def roofline(w: W.Workload, kernel: str, fl: float, by: float, t: float, peaks, tensor_peak: float, burst: bool):
    """Roofline of one kernel: algorithmic FLOPs fl and bytes by over its time t (s), against
    the measured tensor peak (W4A4 expert GEMMs run on the FP4 path: the bf16 peak times the
    nominal dense FP4 / BF16 ratio, 9 / 2.25 PFLOP/s) or the measured copy bandwidth,
    whichever bounds it."""
    fp4_gemm = w.act == "nvfp4" and kernel in ("gate_up_swiglu", "down_sumsq")
    ratio = 4.0 if fp4_gemm else 1.0
    t_tensor = fl / (ratio * tensor_peak * 1e12)
    t_hbm = by / (peaks["hbm_gbs"] * 1e9)
    if t_tensor >= t_hbm:
        roof = {"bound": "tensor", "achieved": fl / t / 1e12, "peak": ratio * tensor_peak, "unit": "TFLOP/s"}
        kind = "burst: max SM clock" if burst else "sustained: below max clock"
        roof["peak_source"] = f"measured bf16 ({kind})" + (" x 4 (FP4 / BF16 nominal)" if fp4_gemm else "")
    else:
        roof = {"bound": "hbm", "achieved": by / t / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "peak_source": "measured copy"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["kernel"] = kernel
    roof["algorithmic_flops"] = fl
    roof["algorithmic_bytes"] = by
    roof["traffic"] = measured_traffic(kernel, w)
    return roof


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


def time_graph(w: W.Workload, model, inp, out, idx, steps: int, warmup: int, world: int, dev, flush_bytes: int = 0):
    """The same forward captured once in a CUDA graph and replayed: CUDA-event time of
    `steps` replays (max over ranks), no host work between launches. flush_bytes > 0: a
    buffer that large is overwritten between replays, outside each replay's own events, and
    the time is the sum of the replays' own durations."""
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
    if flush_bytes:
        flush = torch.empty(flush_bytes // 4, dtype=torch.int32, device=dev)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for i, (a, b_) in enumerate(evs):
            flush.fill_(i)
            a.record(stream)
            graph.replay()
            b_.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        ms = all_max(sum(a.elapsed_time(b_) for a, b_ in evs), world, dev)
    else:
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
             sample_clocks: bool, e2e_steps: int, graph_steps: int = 0, flush_bytes: int = 0):
    """Times `steps` forwards of workload w. flush_bytes > 0: between steps a buffer of that
    many bytes (larger than L2) is overwritten, outside each step's own events, and the step
    time is the sum of the steps' own durations (first to last library event)."""
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
    # the per-kernel breakdown comes from a separate pass with the library recording an
    # event between its launches; the timed steps run the forward exactly as a caller does
    n_inst = min(steps, 10)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nst + 1)] for _ in range(n_inst)]
    for row in ev:
        for e in row:
            e.record(stream)
    handles = [moe.event_handles(row) for row in ev]
    step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
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
    flush = torch.empty(flush_bytes // 4, dtype=torch.int32, device=dev) if flush_bytes else None
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    wall0 = time.time()
    t_start.record(stream)
    for s in range(steps):
        if flush is not None:
            flush.fill_(s)
            step_ev[s][0].record(stream)
        model(inp["x"], out=out, topk_idx=idx)
        if flush is not None:
            step_ev[s][1].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    wall1 = time.time()
    barrier(world)
    if clocks:
        time.sleep(0.2)
        clocks.stop()
    ms = t_start.elapsed_time(t_end)
    if flush is not None:
        ms = sum(a.elapsed_time(b_) for a, b_ in step_ev)
    ms_max = all_max(ms, world, dev)
    code, detail = moe.last_device_status(model.config(w.T, model.workspace))
    if code != 0:
        raise RuntimeError(f"device status {code} detail {detail:#x}")
    # instrumented pass: an event between every launch (same flush between steps)
    for s in range(n_inst):
        if flush is not None:
            flush.fill_(s)
        model(inp["x"], out=out, topk_idx=idx, stage_events=handles[s])
    torch.cuda.synchronize()
    stage_ms = [sum(ev[s][i].elapsed_time(ev[s][i + 1]) for s in range(n_inst)) / n_inst for i in range(nst)]
    # each instrumented step's own duration (its first to its last library event)
    per_step = sorted(ev[s][0].elapsed_time(ev[s][nst]) for s in range(n_inst))
    n_touched = int(torch.unique(idx).numel())
    work = stage_work(w, n_touched)
    dom = max(range(nst), key=lambda i: stage_ms[i])
    dname = stage_names[dom]
    fl, by = work[dname]
    t_dom = stage_ms[dom] * 1e-3
    clk = clocks.summary(wall0, wall1) if clocks else None
    burst = at_full_clock(clk)
    tensor_peak = peaks["bf16_tflops"] if burst else peaks["bf16_tflops_sustained"]
    roof = roofline(w, dname, fl, by, t_dom, peaks, tensor_peak, burst)
    if peak_kind != "measured":
        roof["peak_source"] += " (recipe fallback figures)"
    sf, sb, sf4 = step_work(w, n_touched)
    t_step = ms_max / steps * 1e-3
    bf16_peak = tensor_peak * 1e12
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
    if clk:
        res["clocks"] = clk
    if e2e_steps > 0:
        res["e2e"] = run_e2e(w, model, inp, e2e_steps, world, dev)
    if graph_steps > 0:
        res["graph"] = time_graph(w, model, inp, out, idx, graph_steps, warmup, world, dev, flush_bytes)
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
CPU_TOKENS = 1024


class OracleSample:
    """What the FP64 oracle needs for tokens [0, n) of a workload, generated with the shared
    seeded generator (on the GPU when there is one: the same bytes either way): those x
    rows and the shared weights widened to float64, the routing bias, and the expert
    weights of the experts that routing touches, widened to float64 one expert at a time
    when the oracle asks for them (widen time recorded, so that the timed figure is the
    oracle's arithmetic and not the conversion of 2-byte weights to 8-byte ones)."""

    def __init__(self, w: W.Workload, n_tokens: int, dev):
        import oracle
        self.w, self.n, self.dev = w, n_tokens, dev
        xr = torch.empty((n_tokens, w.D), dtype=W.TORCH_DTYPE[w.dtype], device=dev)
        self.x = oracle.as_f64(W.fill(xr, w.seed, W.TID["x"], 1.0))
        self.shared = {n: oracle.as_f64(W.make_tensor(w, n, dev)) for n in ("W_router", "W_pool", "gamma", "W_unpool")}
        bias = W.zipf_router_bias(w) if w.routing == "zipf" else None
        self.bias = None if bias is None else oracle.as_f64(bias)
        logits = oracle.router_logits(self.x, self.shared["W_router"])
        idx, _, _ = oracle.route(logits, w.k, self.bias)
        self.experts_touched = len(np.unique(idx))
        self.widen_s = 0.0
        self.cache = {}

    def expert(self, e: int):
        if e in self.cache:
            return self.cache[e]
        t0 = time.perf_counter()
        mats = tuple(W.expert_slab(self.w, n, e, self.dev).to(torch.float64).cpu().numpy()
                     for n in ("W_gate", "W_up", "W_down"))
        self.widen_s += time.perf_counter() - t0
        return mats

    def keep_widened(self):
        """Hold every touched expert's float64 weights (for repeated runs), if they fit in
        70% of the host's available memory (the full layer: 103 GB)."""
        need = self.experts_touched * 3 * self.w.L * self.w.I * 8
        try:
            import psutil
            avail = psutil.virtual_memory().available
        except ImportError:
            avail = 0
        if need > 0.7 * avail:
            return False
        import oracle
        logits = oracle.router_logits(self.x, self.shared["W_router"])
        idx, _, _ = oracle.route(logits, self.w.k, self.bias)
        for e in np.unique(idx):
            self.cache[int(e)] = self.expert(int(e))
        return True

    def run(self) -> float:
        """One oracle forward over the sample; returns its time without the widening."""
        import oracle
        w0 = self.widen_s
        t0 = time.perf_counter()
        oracle.latent_moe_forward(self.x, self.shared["W_router"], self.shared["W_pool"], self.expert,
                                  self.shared["gamma"], self.shared["W_unpool"], self.w.k, self.w.eps,
                                  router_bias=self.bias)
        return time.perf_counter() - t0 - (self.widen_s - w0)

    def describe(self) -> str:
        return (f"tokens 0-{self.n - 1} of {self.w.name} ({self.experts_touched} experts), FP64 numpy oracle "
                f"expert-major, f64 widening untimed")


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def blas_threads() -> int:
    """Threads the host BLAS runs the oracle's matrix products on."""
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except ImportError:
        pass
    return host_cores()


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
    sample = OracleSample(w, n_tokens, dev)
    dt = sample.run()
    flops_per_token = 2 * (w.E * w.D + w.L * w.D + w.k * 3 * w.L * w.I + w.D * w.L)
    return {"value": n_tokens / dt, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": sample.describe() + f"; {dt:.1f} s, {n_tokens * flops_per_token / dt / 1e9:.0f} GFLOP/s"}


def run_reference(w: W.Workload, args, dev):
    """The FP64 oracle as the reference arm, on the same basis as cpu_baseline: every step
    runs the block on tokens 0..CPU_TOKENS-1 of the workload, expert-major, with the expert
    weights widened to float64 outside the timed region (held across steps when they fit in
    host memory, else widened again each step, untimed)."""
    sample = OracleSample(w, args.cpu_tokens, dev)
    sample.keep_widened()
    times = [sample.run() for _ in range(args.warmup + args.steps)][args.warmup:]
    total = sum(times)
    value = args.steps * sample.n / total
    return {
        "metric": metric_name(), "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(w), "impl": "reference",
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": sample.describe() + " (each step)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ------------------------------------------------------------------------------ plumbing
def metric_name():
    return "latent-MoE layer tokens/s on 1 B200 (T=8192 prefill, T=64 decode); % roofline"


def config_dict(w: W.Workload):
    """The workload named by what it is; the same dict in both arms."""
    return {"workload": f"{w.name}: latent-MoE layer T={w.T} D={w.D} L={w.L} I={w.I} E={w.E} top-{w.k} "
                        f"{w.dtype} {w.routing}",
            "l2": "inputs > L2 (weights streamed)"}


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


def sig(v, n=4):
    """v rounded to n significant digits (keeps the JSON line short)."""
    if v is None or v == 0 or not math.isfinite(v):
        return v
    return round(v, n - 1 - int(math.floor(math.log10(abs(v)))))


SIDE_FIELDS = ["tokens/s", "ms/step", "dominant kernel roofline frac", "graph ms/step"]


def side_entry(r):
    """One side workload in the JSON line, as the list SIDE_FIELDS names (the graph-replay
    time only where the workload is also timed that way)."""
    e = [sig(r["value"]), sig(r["ms_per_step"]), sig(r["roofline"]["frac"], 3)]
    if "graph" in r:
        e.append(sig(r["graph"]["ms_per_step"]))
    return e


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="prefill", choices=list(W.WORKLOADS))
    ap.add_argument("--no-side", action="store_true", help="skip the side workloads")
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle cpu_baseline")
    ap.add_argument("--no-nvfp4", action="store_true", help="skip the NVFP4-expert side workloads")
    ap.add_argument("--cpu-tokens", type=int, default=CPU_TOKENS)
    ap.add_argument("--detail", default=None, help="also write every measurement (per-kernel times, "
                                                   "rooflines of every workload) to this JSON file")
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
            print(json.dumps(run_reference(W.WORKLOADS[args.workload], args, dev), separators=(",", ":")), flush=True)
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

        def run(wl, inputs, steps, **kw):
            return run_ours(wl, inputs, steps, args.warmup, rank, world, peaks, peak_kind, True, **kw)
        main_res = run(w, inp, args.steps, e2e_steps=min(args.steps, 20),
                       graph_steps=args.steps if w.name.endswith("decode") else 0)
        side = {}
        if not args.no_side and w.name == "prefill":
            wd = W.WORKLOADS["decode"]
            inp_d = dict(inp, x=rank_tokens(wd, rank, dev))
            side["decode"] = run(wd, inp_d, max(args.steps, 50), e2e_steps=0, graph_steps=max(args.steps, 50))
            wz = W.WORKLOADS["prefill_zipf"]
            side["prefill_zipf"] = run(wz, dict(inp, router_bias=W.zipf_router_bias(wz).to(dev)), args.steps,
                                       e2e_steps=0)
            # the whole feed-forward sublayer: pre-norm, the block, post-norm, residual gate
            side["prefill_sublayer"] = run(w, dict(inp, **W.sublayer_inputs(w, dev)), args.steps, e2e_steps=0)
            if not args.no_nvfp4:
                # NVFP4 experts (quantised from the same bf16 weights): T=4096 and a T=64 decode
                wq = W.WORKLOADS["nvfp4"]
                q = W.make_inputs(wq, dev, names=["W_gate", "W_up", "W_down"])
                inp_q = dict({k: v for k, v in inp.items() if k not in ("W_gate", "W_up", "W_down")}, **q)
                inp_q["x"] = rank_tokens(wq, rank, dev)
                side["nvfp4"] = run(wq, inp_q, args.steps, e2e_steps=0)
                wqd = W.WORKLOADS["nvfp4_decode"]
                inp_qd = dict(inp_q, x=rank_tokens(wqd, rank, dev))
                side["nvfp4_decode"] = run(wqd, inp_qd, max(args.steps, 50), e2e_steps=0,
                                           graph_steps=max(args.steps, 50))
                # the same weights with NVFP4 activations (W4A4, tcgen05 kind::mxf4nvf4)
                side["nvfp4_w4a4"] = run(W.WORKLOADS["nvfp4_w4a4"], inp_q, args.steps, e2e_steps=0)
                side["nvfp4_w4a4_decode"] = run(W.WORKLOADS["nvfp4_w4a4_decode"], inp_qd, max(args.steps, 50),
                                                e2e_steps=0, graph_steps=max(args.steps, 50))
                del q, inp_q, inp_qd
            # the mid layer (0.41 GB of weights): a 256 MiB buffer is overwritten between steps
            # so that no step finds the previous one's weights in L2
            del inp_d
            wm = W.WORKLOADS["mid"]
            inp_m = make_rank_inputs(wm, rank, dev)
            side["mid"] = run(wm, inp_m, max(args.steps, 50), e2e_steps=0, flush_bytes=256 << 20,
                              graph_steps=max(args.steps, 50))
        if rank == 0:
            roof = {k: main_res["roofline"][k] for k in ("bound", "achieved", "peak", "unit", "frac", "traffic",
                                                          "kernel", "peak_source")}
            for k in ("achieved", "peak", "frac"):
                roof[k] = sig(roof[k])
            clk = main_res.get("clocks") or {}
            line = {
                "metric": metric_name(), "value": sig(main_res["value"], 6), "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": sig(main_res["ms_per_step"], 5),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
                "data": "synthetic",
                "config": config_dict(w), "roofline": roof,
                "step_roofline_frac": sig(main_res["step"]["frac_of_step_roofline"], 3),
                "gpu_launches": main_res["gpu_launches"],
                "clocks": {"sm_mhz": clk.get("sm_mhz"), "sm_max_mhz": clk.get("sm_max_mhz"),
                           "reasons": clk.get("reasons", [])},
            }
            e2e = main_res.get("e2e")
            if e2e:
                line["e2e"] = {"value": sig(e2e["value"], 6), "unit": e2e["unit"],
                               "h2d_bytes_per_step": e2e["h2d_bytes_per_step"],
                               "d2h_bytes_per_step": e2e["d2h_bytes_per_step"]}
            if "graph" in main_res:
                line["graph_replay_ms"] = sig(main_res["graph"]["ms_per_step"])
            if side:
                line["side_fields"] = SIDE_FIELDS
                line["side"] = {name: side_entry(r) for name, r in side.items()}
            if world == 1 and not args.no_cpu:
                line["cpu_baseline"] = cpu_baseline(w, dev, args.cpu_tokens)
            if args.detail:
                detail = {"line": line, "main": main_res, "side": side, "cpu_model": cpu_model()}
                with open(args.detail, "w") as f:
                    json.dump(detail, f, indent=1, default=float)
            print(json.dumps(line, separators=(",", ":")), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
