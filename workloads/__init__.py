"""Seeded synthetic inputs for the latent-MoE block, and the named workload presets.

This module is shared by the two sides that must see identical bytes: the CUDA path
(tests, bench) and the FP64 oracle. It holds no arithmetic of the method itself, only
a counter-based normal generator and the shapes of the workloads:

* every element is a pure function of (seed, tensor id, flat element index), so any slab
  of a tensor (one expert's weights, a few token rows) can be regenerated on its own,
  on the CPU or on the GPU, without generating the rest;
* the 64-bit counter hash is the SplitMix64 finaliser (Steele, Lea and Flood, "Fast
  splittable pseudorandom number generators", OOPSLA 2014); two hashes give two
  uniforms, and the Box-Muller transform turns them into one N(0,1) draw in float64;
* the float64 draw times the tensor's standard deviation is rounded once to the
  workload's storage dtype (float32 or bfloat16, round-to-nearest-even by torch).

Shapes come from the Muse Spark Open deep dive, §4.1 table (256 experts, top-8,
hidden 8192, latent 4096, SwiGLU 4096 -> 2x4096 -> 4096) and from the five workload
descriptions of this project (tiny, mid, decode, prefill uniform / Zipf-skewed).
Weights are N(0, 1/fan_in); gamma is N(0, 0.1) read as variance 0.1; x is N(0, 1).
"""
from __future__ import annotations

import dataclasses
import math
import os
from typing import Dict, Optional

import torch

# ----------------------------------------------------------------------------------------
# workload presets
# ----------------------------------------------------------------------------------------


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int          # tokens
    D: int          # hidden width (router and pooler input, unpooler output)
    L: int          # latent width (expert input and output)
    I: int          # expert intermediate width
    E: int          # experts
    k: int          # experts per token
    dtype: str      # storage / activation dtype: "f32" or "bf16"
    eps: float = 1e-6
    routing: str = "uniform"   # "uniform" (no bias) or "zipf" (selection bias, s=1.2)
    seed: int = 0
    experts: str = "bf16"      # expert weight storage: "bf16" (the dtype) or "nvfp4"
    act: str = "bf16"          # expert GEMM activations: "bf16" or "nvfp4" (W4A4)

    def with_tokens(self, T: int) -> "Workload":
        return dataclasses.replace(self, T=T)


WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", T=16, D=256, L=128, I=128, E=8, k=2, dtype="f32"),
    "mid": Workload("mid", T=256, D=2048, L=1024, I=1024, E=64, k=4, dtype="bf16"),
    "decode": Workload("decode", T=64, D=8192, L=4096, I=4096, E=256, k=8, dtype="bf16"),
    "prefill": Workload("prefill", T=8192, D=8192, L=4096, I=4096, E=256, k=8, dtype="bf16"),
    "prefill_zipf": Workload("prefill_zipf", T=8192, D=8192, L=4096, I=4096, E=256, k=8,
                             dtype="bf16", routing="zipf"),
    # full-width layer with 16 experts and 256 tokens per expert: the prefill tile
    # shapes on ~2 GB of device memory (profiling captures)
    "prefill_e16": Workload("prefill_e16", T=2048, D=8192, L=4096, I=4096, E=16, k=2, dtype="bf16"),
    # full layer with NVFP4 expert weights (router, pooler, unpooler and activations bf16)
    "nvfp4": Workload("nvfp4", T=4096, D=8192, L=4096, I=4096, E=256, k=8, dtype="bf16", experts="nvfp4"),
    "nvfp4_decode": Workload("nvfp4_decode", T=64, D=8192, L=4096, I=4096, E=256, k=8, dtype="bf16",
                             experts="nvfp4"),
    # decode-like NVFP4 case on ~1 GB of weights (2-3 tokens per expert; profiling captures)
    "nvfp4_decode_e32": Workload("nvfp4_decode_e32", T=32, D=8192, L=4096, I=4096, E=32, k=2, dtype="bf16",
                                 experts="nvfp4"),
    # NVFP4 experts on prefill-sized tiles (256 tokens per expert) at a few GB: the small case
    # the W4A16 kernel is profiled on
    "nvfp4_e16": Workload("nvfp4_e16", T=2048, D=8192, L=4096, I=4096, E=16, k=2, dtype="bf16", experts="nvfp4"),
    # the same NVFP4 layers with both operands of the expert GEMMs in NVFP4 (W4A4)
    "nvfp4_w4a4": Workload("nvfp4_w4a4", T=4096, D=8192, L=4096, I=4096, E=256, k=8, dtype="bf16",
                           experts="nvfp4", act="nvfp4"),
    "nvfp4_w4a4_decode": Workload("nvfp4_w4a4_decode", T=64, D=8192, L=4096, I=4096, E=256, k=8, dtype="bf16",
                                  experts="nvfp4", act="nvfp4"),
}

# tensor ids of the generator (fixed, part of the workload definition)
TID = {"x": 1, "W_router": 2, "W_pool": 3, "W_gate": 4, "W_up": 5, "W_down": 6,
       "gamma": 7, "W_unpool": 8, "zipf_rank": 10}


def shapes(w: Workload) -> Dict[str, tuple]:
    """Row-major shapes, weights stored [out, in] like a bias-free linear layer."""
    return {
        "x": (w.T, w.D),
        "W_router": (w.E, w.D),
        "W_pool": (w.L, w.D),
        "W_gate": (w.E, w.I, w.L),
        "W_up": (w.E, w.I, w.L),
        "W_down": (w.E, w.L, w.I),
        "gamma": (w.E, w.L),
        "W_unpool": (w.D, w.L),
    }


def stddev(w: Workload, name: str) -> float:
    fan_in = {"x": None, "W_router": w.D, "W_pool": w.D, "W_gate": w.L, "W_up": w.L,
              "W_down": w.I, "gamma": None, "W_unpool": w.L}[name]
    if name == "x":
        return 1.0
    if name == "gamma":
        return math.sqrt(0.1)
    return 1.0 / math.sqrt(fan_in)


TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}

# ----------------------------------------------------------------------------------------
# counter-based generator
# ----------------------------------------------------------------------------------------

_M64 = (1 << 64) - 1


def _s64(v: int) -> int:
    """Two's-complement view of a 64-bit constant, for torch int64 arithmetic."""
    v &= _M64
    return v - (1 << 64) if v >= (1 << 63) else v


_GOLDEN = _s64(0x9E3779B97F4A7C15)
_MIX1 = _s64(0xBF58476D1CE4E5B9)
_MIX2 = _s64(0x94D049BB133111EB)
_TIDMUL = _s64(0xD1B54A32D192ED03)


def _lsr(z: torch.Tensor, s: int) -> torch.Tensor:
    # logical right shift of the 64-bit pattern held in a signed int64 tensor
    return (z >> s) & ((1 << (64 - s)) - 1)


def _splitmix_finalise(z: torch.Tensor) -> torch.Tensor:
    z = z ^ _lsr(z, 30)
    z = z * _MIX1
    z = z ^ _lsr(z, 27)
    z = z * _MIX2
    return z ^ _lsr(z, 31)


def _stream_base(seed: int, tid: int) -> int:
    return _s64((seed * 0x9E3779B97F4A7C15 + tid * 0xD1B54A32D192ED03) & _M64)


def normal_f64(seed: int, tid: int, start: int, count: int,
               device: torch.device | str = "cpu") -> torch.Tensor:
    """N(0,1) draws for flat element indices [start, start+count) of tensor `tid`."""
    idx = torch.arange(start, start + count, dtype=torch.int64, device=device)
    ctr = idx * 2 + _stream_base(seed, tid)
    h1 = _splitmix_finalise(ctr * _GOLDEN)
    h2 = _splitmix_finalise((ctr + 1) * _GOLDEN)
    u1 = (_lsr(h1, 11).to(torch.float64) + 0.5) * (2.0 ** -53)   # (0, 1)
    u2 = _lsr(h2, 11).to(torch.float64) * (2.0 ** -53)           # [0, 1)
    return torch.sqrt(-2.0 * torch.log(u1)) * torch.cos((2.0 * math.pi) * u2)


def uniform_u64(seed: int, tid: int, count: int) -> torch.Tensor:
    """Raw 64-bit hashes (as int64) of indices 0..count-1 of stream `tid` (CPU)."""
    idx = torch.arange(count, dtype=torch.int64)
    return _splitmix_finalise((idx * 2 + _stream_base(seed, tid)) * _GOLDEN)


def fill(out: torch.Tensor, seed: int, tid: int, std: float, start: int = 0,
         chunk: int = 1 << 25) -> torch.Tensor:
    """Fill `out` (any dtype, contiguous) with std*N(0,1) of elements [start, start+numel)."""
    flat = out.view(-1)
    n = flat.numel()
    for off in range(0, n, chunk):
        m = min(chunk, n - off)
        flat[off:off + m] = (normal_f64(seed, tid, start + off, m, out.device) * std).to(out.dtype)
    return out


def make_tensor(w: Workload, name: str, device="cpu", dtype: Optional[torch.dtype] = None,
                chunk: int = 1 << 25) -> torch.Tensor:
    dt = dtype if dtype is not None else TORCH_DTYPE[w.dtype]
    t = torch.empty(shapes(w)[name], dtype=dt, device=device)
    return fill(t, w.seed, TID[name], stddev(w, name), chunk=chunk)


def expert_slab(w: Workload, name: str, e: int, device="cpu",
                dtype: Optional[torch.dtype] = None) -> torch.Tensor:
    """Expert e's [out, in] matrix of W_gate / W_up / W_down, generated on its own."""
    shp = shapes(w)[name]
    per = shp[1] * shp[2]
    dt = dtype if dtype is not None else TORCH_DTYPE[w.dtype]
    t = torch.empty(shp[1:], dtype=dt, device=device)
    return fill(t, w.seed, TID[name], stddev(w, name), start=e * per)


SUBLAYER_TID = {"ffn_pre_gain": 13, "ffn_post_gain": 14, "residual_gate": 15}


def sublayer_inputs(w: Workload, device="cpu") -> Dict[str, torch.Tensor]:
    """Parameters of the feed-forward sublayer around the block: the pre- and post-norm
    gain offsets [D] ~ N(0, 0.1) (variance, like gamma) in the workload dtype, and the
    residual gate's parameters g [D] ~ N(0, 1) in float32 -- wider than the N(0, 0.02^2)
    initialisation the pages quote, so that beta spans (0, 1) and some channels reach
    the alpha^2 floor (g > 2.28)."""
    out = {}
    for n in ("ffn_pre_gain", "ffn_post_gain"):
        t = torch.empty((w.D,), dtype=TORCH_DTYPE[w.dtype], device=device)
        out[n] = fill(t, w.seed, SUBLAYER_TID[n], math.sqrt(0.1))
    g = torch.empty((w.D,), dtype=torch.float32, device=device)
    out["residual_gate"] = fill(g, w.seed, SUBLAYER_TID["residual_gate"], 1.0)
    return out


def make_inputs(w: Workload, device="cpu", names=None) -> Dict[str, torch.Tensor]:
    """The workload's tensors. For NVFP4 experts, W_gate / W_up / W_down are replaced by
    <name>_codes, <name>_scales and <name>_mscale (see quantize_nvfp4), each expert
    quantised from the same bf16 weights a bf16 workload would use."""
    names = names or list(shapes(w).keys())
    out = {}
    for n in names:
        if w.experts == "nvfp4" and n in ("W_gate", "W_up", "W_down"):
            out.update(make_nvfp4_experts(w, n, device))
        else:
            out[n] = make_tensor(w, n, device)
    if w.routing == "zipf":
        out["router_bias"] = zipf_router_bias(w).to(device)
    return out


# ----------------------------------------------------------------------------------------
# NVFP4 expert weights: 4-bit E2M1 values, one E4M3 scale per 16 weights of a row, one
# float32 scale per expert matrix (the format the deep dive's §7.4 describes). The
# quantiser is part of input generation; any quantiser would do for parity, since both
# sides read the same codes.
# ----------------------------------------------------------------------------------------
_E2M1_MIDPOINTS = (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)
_E2M1_TIES_UP = (0.75, 1.75, 3.5)   # midpoints whose upper neighbour has the even mantissa


def _e2m1_codes(q: torch.Tensor) -> torch.Tensor:
    """Round to nearest E2M1 value (ties to even), saturating at +-6; returns codes 0..15."""
    a = q.abs().clamp(max=6.0)
    mag = torch.zeros_like(a, dtype=torch.uint8)
    for mid in _E2M1_MIDPOINTS:
        mag += (a > mid).to(torch.uint8)
    for mid in _E2M1_TIES_UP:
        mag += (a == mid).to(torch.uint8)
    return mag | (torch.signbit(q).to(torch.uint8) << 3)


def quantize_nvfp4(wt: torch.Tensor):
    """[out, in] weights -> (codes uint8 [out, in/2] low nibble first, block scales uint8
    E4M3 [out, in/16], matrix scale float). Matrix scale amax/(6*448); block scale
    E4M3(amax_block / (6 * matrix scale)); code E2M1(w / (block * matrix scale))."""
    x = wt.to(torch.float32)
    out_dim, in_dim = x.shape
    amax = float(x.abs().max())
    ms = amax / (6.0 * 448.0) if amax > 0 else 1.0
    blocks = x.view(out_dim, in_dim // 16, 16)
    bscale = (blocks.abs().amax(-1) / (6.0 * ms)).clamp(max=448.0).to(torch.float8_e4m3fn)
    denom = bscale.to(torch.float32) * ms
    q = torch.where(denom[..., None] > 0, blocks / denom[..., None].clamp(min=1e-30), torch.zeros_like(blocks))
    codes = _e2m1_codes(q).view(out_dim, in_dim // 2, 2)
    packed = codes[..., 0] | (codes[..., 1] << 4)
    return packed.contiguous(), bscale.view(torch.uint8).contiguous(), ms


def make_nvfp4_experts(w: Workload, name: str, device="cpu") -> Dict[str, torch.Tensor]:
    shp = shapes(w)[name]
    E, rows, cols = shp
    codes = torch.empty((E, rows, cols // 2), dtype=torch.uint8, device=device)
    scales = torch.empty((E, rows, cols // 16), dtype=torch.uint8, device=device)
    mscale = torch.empty(E, dtype=torch.float32, device=device)
    for e in range(E):
        c, s, m = quantize_nvfp4(expert_slab(w, name, e, device))
        codes[e], scales[e], mscale[e] = c, s, m
    return {f"{name}_codes": codes, f"{name}_scales": scales, f"{name}_mscale": mscale}



# ----------------------------------------------------------------------------------------
# Zipf-skewed routing (selection bias), stored input
# ----------------------------------------------------------------------------------------

_HERE = os.path.dirname(os.path.abspath(__file__))


def zipf_target_loads(T: int, E: int, k: int, s: float = 1.2) -> torch.Tensor:
    """Water-filled Zipf(s) target token count per popularity rank r = 1..E.

    A pure Zipf share for rank 1 exceeds 1/k of all assignments (an expert cannot take a
    token twice), so loads are capped at T and the excess is spread over the other ranks
    in proportion to r^-s until every cap holds and the loads sum to T*k.
    """
    r = torch.arange(1, E + 1, dtype=torch.float64)
    wgt = r ** (-s)
    total = float(T * k)
    capped = torch.zeros(E, dtype=torch.bool)
    loads = torch.zeros(E, dtype=torch.float64)
    for _ in range(E):
        free = ~capped
        rest = total - T * int(capped.sum())
        loads = torch.where(capped, torch.full_like(loads, float(T)), rest * wgt / wgt[free].sum())
        new_cap = loads > T
        if not bool((new_cap & ~capped).any()):
            break
        capped = capped | new_cap
    return torch.clamp(loads, max=float(T))


def zipf_rank_to_expert(w: Workload) -> torch.Tensor:
    """Seeded permutation: expert id that holds popularity rank r (0-based)."""
    h = uniform_u64(w.seed, TID["zipf_rank"], w.E)
    return torch.argsort(h, stable=True)


def zipf_bias_path(w: Workload) -> str:
    return os.path.join(_HERE, f"zipf_router_bias_T{w.T}_E{w.E}_k{w.k}_D{w.D}_seed{w.seed}.txt")


def zipf_router_bias(w: Workload) -> torch.Tensor:
    """The stored selection bias (float32 [E]) that skews routing to the Zipf target.

    Written by workloads/calibrate_zipf_bias.py; both the CUDA path and the oracle read
    these same 256 numbers.
    """
    path = zipf_bias_path(w)
    if not os.path.exists(path):
        raise FileNotFoundError(f"{path} missing: run python -m workloads.calibrate_zipf_bias")
    vals = [float(line.split()[1]) for line in open(path) if line.strip() and not line.startswith("#")]
    if len(vals) != w.E:
        raise ValueError(f"{path}: expected {w.E} values, got {len(vals)}")
    return torch.tensor(vals, dtype=torch.float32)
