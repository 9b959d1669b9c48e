"""Helpers of the GPU parity tests: run the CUDA path through the C ABI, run the FP64
oracle on the same bytes, and compare with the tolerances the block is held to.

Tolerances (for every workload):
  * expert indices: the selected SET must equal the oracle's exactly, except for tokens
    whose k-th and (k+1)-th oracle keys differ by less than TIE_TOL; for those the GPU
    set must be one of the oracle's own valid alternatives, and the oracle output for
    that alternative is the reference. The ORDER inside the set must be non-increasing
    in the oracle's keys up to TIE_TOL (several orders are correct for near-equal keys);
  * routing weights: |g_gpu - g_oracle| <= 2e-4 per selected expert;
  * outputs: relative L2 error <= 1e-2 and max-abs error <= 5e-2 * rms(out).
"""
from __future__ import annotations

import math
from typing import Dict, Optional, Sequence

import numpy as np
import torch

import latent_mixture_experts_moe_b200 as moe
import oracle
import workloads as W

TIE_TOL = 1e-4
G_TOL = 2e-4
REL_L2 = 1e-2
MAX_ABS_RMS = 5e-2


def rel_l2(got: np.ndarray, ref: np.ndarray) -> float:
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


def assert_close(got: np.ndarray, ref: np.ndarray, what: str, rel=REL_L2, max_abs_rms=MAX_ABS_RMS):
    got = np.asarray(got, dtype=np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    r = rel_l2(got, ref)
    rms = math.sqrt(float(np.mean(ref * ref)))
    ma = float(np.abs(got - ref).max())
    assert r <= rel, f"{what}: rel-L2 {r:.3e} > {rel}"
    assert ma <= max_abs_rms * rms, f"{what}: max-abs {ma:.3e} > {max_abs_rms} * rms {rms:.3e}"
    return r, ma / rms


def assert_close_stored(got: np.ndarray, ref: np.ndarray, what: str, rel=REL_L2, max_abs_rms=MAX_ABS_RMS,
                        stored_bits: int = 8):
    """For an intermediate the CUDA path stores in a narrow type (bf16: 8 significant bits)
    and the oracle never rounds: rel-L2 <= rel, and elementwise |got - ref| <= max_abs_rms *
    rms(ref) + 2^-stored_bits * |ref| -- the block-output bound plus one unit in the last
    place of the stored value itself (its own rounding, and the neighbour a value within
    the computational error of a rounding boundary may round to). Large elements of an
    intermediate (a latent row dominated by one expert's normalised output reaches |c| ~ 10,
    where a bf16 unit is 2^-4) would otherwise fail a bound meant for the block output."""
    got = np.asarray(got, dtype=np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    r = rel_l2(got, ref)
    rms = math.sqrt(float(np.mean(ref * ref)))
    excess = np.abs(got - ref) - (max_abs_rms * rms + np.ldexp(np.abs(ref), -stored_bits))
    assert r <= rel, f"{what}: rel-L2 {r:.3e} > {rel}"
    worst = int(np.argmax(excess))
    assert excess.flat[worst] <= 0, (f"{what}: element {np.unravel_index(worst, ref.shape)} got "
                                     f"{got.flat[worst]:.6g} ref {ref.flat[worst]:.6g} (rms {rms:.3e})")
    return r, float(np.abs(got - ref).max()) / rms


def ws_view(ws: torch.Tensor, off: int, dtype: torch.dtype, shape: Sequence[int]) -> torch.Tensor:
    n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
    return ws[off:off + n].view(dtype).view(*shape)


class Run:
    """One forward of the CUDA path with its routing outputs and workspace (modes: the
    keyword arguments of latent_mixture_experts_moe_b200.make_config)."""

    def __init__(self, w: W.Workload, inp: Dict[str, torch.Tensor], T: Optional[int] = None, **modes):
        T = T or w.T
        self.w, self.T = w, T
        weights = {k: v for k, v in inp.items() if k != "x"}
        if w.act == "nvfp4":
            modes = dict(modes, act_format=moe.ACT_NVFP4)
        self.model = moe.LatentMoE(weights, T_max=T, k=w.k, eps=w.eps, **modes)
        dev = inp["x"].device
        self.idx = torch.full((T, w.k), -1, dtype=torch.int32, device=dev)
        self.g = torch.zeros((T, w.k), dtype=torch.float32, device=dev)
        self.out = self.model(inp["x"][:T], topk_idx=self.idx, topk_w=self.g)
        torch.cuda.synchronize()
        cfg = self.model.config(T, self.model.workspace)
        code, detail = moe.last_device_status(cfg)
        assert code == 0, f"device status {moe.STATUS.get(code)} detail {detail:#x}"
        self.layout = moe.workspace_layout(cfg)

    def inter(self, name: str, dtype, shape):
        return ws_view(self.model.workspace, self.layout[name], dtype, shape)

    def act(self):
        return torch.float32 if self.w.dtype == "f32" else torch.bfloat16


def host(t: torch.Tensor) -> np.ndarray:
    return oracle.as_f64(t)


def expert_source(inp: Dict[str, torch.Tensor]):
    if "W_gate_codes" in inp:
        # NVFP4 experts: the oracle runs on exactly the dequantised codes
        def deq(name, e):
            return oracle.dequantize_nvfp4(inp[name + "_codes"][e].cpu().numpy(), inp[name + "_scales"][e].cpu().numpy(),
                                           float(inp[name + "_mscale"][e]))
        return lambda e: (deq("W_gate", e), deq("W_up", e), deq("W_down", e))
    return lambda e: (inp["W_gate"][e], inp["W_up"][e], inp["W_down"][e])


def w4a4_reference(run: "Run", rows: np.ndarray):
    """For the W4A4 oracle: the CUDA path's quantised activation rows of each assignment, as
    candidate decisions that the oracle adopts only where its own input sits at a rounding
    boundary (oracle.quantize_activations_nvfp4 raises on any other difference)."""
    k, L, I, R = run.w.k, run.w.L, run.w.I, run.layout["rows"]
    ginv = run.inter("inv", torch.int32, (run.T * k,)).cpu().numpy()
    zc = run.inter("zq_codes", torch.uint8, (R, L // 2)).cpu().numpy()
    zs = run.inter("zq_scales", torch.uint8, (R, L // 16)).cpu().numpy()
    hc = run.inter("hq_codes", torch.uint8, (R, I // 2)).cpu().numpy()
    hs = run.inter("hq_scales", torch.uint8, (R, I // 16)).cpu().numpy()

    def ref(tok, slot):
        r = ginv[np.asarray(rows)[tok] * k + slot]
        return (zc[r], zs[r]), (hc[r], hs[r])
    return ref


def oracle_block(w: W.Workload, inp: Dict[str, torch.Tensor], rows: np.ndarray, run: Optional["Run"] = None,
                 **kw) -> Dict[str, np.ndarray]:
    """The oracle on token rows `rows` of x (tokens are independent). For W4A4 workloads,
    `run` supplies the candidate quantisation decisions (w4a4_reference)."""
    x = host(inp["x"][torch.as_tensor(rows, device=inp["x"].device)])
    bias = host(inp["router_bias"]) if "router_bias" in inp else None
    if "pre_norm_gain" in inp:
        kw = dict(kw, pre_norm_gain=host(inp["pre_norm_gain"]))
    for name, key in (("ffn_pre_gain", "ffn_pre_gain"), ("ffn_post_gain", "ffn_post_gain"), ("residual_gate", "gate")):
        if name in inp:
            kw = dict(kw, **{key: host(inp[name])})
    if "ffn_pre_gain" in inp and w.dtype == "bf16":
        kw = dict(kw, xn_round="bf16")
    if w.act == "nvfp4":
        kw = dict(kw, act_format="nvfp4")
        if run is not None:
            kw = dict(kw, act_ref=w4a4_reference(run, rows))
    return oracle.latent_moe_forward(x, host(inp["W_router"]), host(inp["W_pool"]), expert_source(inp),
                                     host(inp["gamma"]), host(inp["W_unpool"]), w.k, w.eps, router_bias=bias,
                                     **kw)


def check_routing(ref: Dict[str, np.ndarray], gpu_idx: np.ndarray, gpu_g: np.ndarray, k: int):
    """Returns the tokens whose GPU set is a valid alternative different from the oracle's
    (near ties), after checking every token's set, order and weights."""
    keys, ridx, rg = ref["keys"], ref["idx"], ref["g"]
    alt_tokens = []
    for t in range(gpu_idx.shape[0]):
        gs, rs = set(gpu_idx[t].tolist()), set(ridx[t].tolist())
        assert len(gs) == k, f"token {t}: repeated expert in {gpu_idx[t]}"
        if gs != rs:
            srt = np.sort(keys[t])[::-1]
            gap = srt[k - 1] - srt[k] if k < keys.shape[1] else np.inf
            assert gap < TIE_TOL, f"token {t}: GPU {sorted(gs)} vs oracle {sorted(rs)}, gap {gap:.2e}"
            assert tuple(sorted(gs)) in oracle.topk_alternatives(keys[t], k, TIE_TOL), f"token {t}"
            alt_tokens.append(t)
        ko = keys[t][gpu_idx[t]]
        assert np.all(np.diff(ko) <= TIE_TOL), f"token {t}: order {gpu_idx[t]} keys {ko}"
        if gs == rs:
            for j in range(k):
                e = gpu_idx[t, j]
                jr = int(np.nonzero(ridx[t] == e)[0][0])
                assert abs(gpu_g[t, j] - rg[t, jr]) <= G_TOL, f"token {t} expert {e}: g {gpu_g[t, j]} vs {rg[t, jr]}"
    return alt_tokens


def oracle_on_gpu_alternatives(w, inp, rows, ref, gpu_idx, alt_tokens, run=None, **kw):
    """For near-tie tokens, the oracle output under the oracle's alternative routing that
    the GPU chose (found in oracle.topk_alternatives), with the oracle's own weights."""
    out = ref["out"].copy()
    for t in alt_tokens:
        sel = np.array(sorted(gpu_idx[t].tolist(), key=lambda e: (-ref["keys"][t][e], e)))[None, :]
        if kw.get("router_mode", "softmax") == "sigmoid":
            g = oracle.sigmoid_weights(ref["logits"][t:t + 1], sel, kw.get("logit_scale", 1.0),
                                       kw.get("routed_scaling", 1.0))
        else:
            g = oracle.softmax_weights(ref["logits"][t:t + 1], sel)
        r1 = oracle_block(w, inp, rows[t:t + 1], run=run, routing=(sel, g), **kw)
        out[t] = r1["out"][0]
    return out


def forced_weights(logits: np.ndarray, idx: np.ndarray, router_mode: str = "softmax", logit_scale: float = 1.0,
                   routed_scaling: float = 1.0, **_) -> np.ndarray:
    """The oracle's routing weights for the experts idx[t, :] of every token (any valid
    set and order): its own weights where idx is its own choice, the weights of the
    alternative set where a near tie let the CUDA path pick another valid set."""
    if router_mode == "sigmoid":
        return oracle.sigmoid_weights(logits, idx, logit_scale, routed_scaling)
    return oracle.softmax_weights(logits, idx)


def check_every_token(w: W.Workload, inp: Dict[str, torch.Tensor], run: "Run", rel: float = REL_L2,
                      **oracle_modes) -> Dict[str, float]:
    """Whole-output parity of one forward at any size (the benchmark spec tolerances):

    * routing: every token's set, order and weights against the oracle's router on all
      tokens (check_routing: a differing set only at a near tie, and then one of the
      oracle's valid alternatives);
    * the oracle then runs the whole block on every token under the CUDA path's validated
      routing (its sets and slot order, the oracle's weights for them), so that every
      assignment row has a reference: out [T, D], the pooler's z, the expert outputs y and
      their sums of squares on every one of the T*k rows, and the combined latent c;
    * the permutation (counts, padded offsets, inv, row_token) bit for bit against its
      integer definition on the CUDA path's (validated) expert indices.
    The output is held to assert_close (the block's tolerance); the intermediates the CUDA
    path stores in the activation dtype (z, y, c) to assert_close_stored, and the sums of
    squares (float32 partials) to twice the relative tolerance.
    Returns the measured errors and the near-tie count."""
    T, k, L, E = run.T, w.k, w.L, w.E
    rows = np.arange(T)
    x = host(inp["x"][:T])
    logits = oracle.router_logits(x, host(inp["W_router"]))
    del x
    bias = host(inp["router_bias"]) if "router_bias" in inp else None
    ro = {n: oracle_modes[n] for n in ("router_mode", "logit_scale", "routed_scaling") if n in oracle_modes}
    idx, g, keys = oracle.route(logits, k, bias, **ro)
    gidx = run.idx.cpu().numpy()
    alts = check_routing({"keys": keys, "idx": idx, "g": g}, gidx, run.g.cpu().numpy(), k)
    routing = (gidx.astype(np.int64), forced_weights(logits, gidx, **ro))
    del logits, keys
    ref = oracle_block(w, inp, rows, run=run, routing=routing, **oracle_modes)
    res = {"near_ties": len(alts)}
    res["out"], _ = assert_close(host(run.out), ref.pop("out"), f"{w.name} out (all {T} tokens)", rel=rel)
    act = run.act()
    bits = 8 if act == torch.bfloat16 else 24
    res["z"], _ = assert_close_stored(host(run.inter("z", act, (T, L))), ref.pop("z"), f"{w.name} z", rel=rel,
                                      stored_bits=bits)
    res["c"], _ = assert_close_stored(host(run.inter("c", act, (T, L))), ref.pop("c"), f"{w.name} c", rel=rel,
                                      stored_bits=bits)
    # the permutation, from the validated indices
    counts, offsets, inv = expected_permutation(gidx, E)
    R = run.layout["rows"]
    assert np.array_equal(run.inter("expert_count", torch.int32, (E,)).cpu().numpy(), counts)
    assert np.array_equal(run.inter("expert_offset", torch.int32, (E + 1,)).cpu().numpy(), offsets)
    ginv = run.inter("inv", torch.int32, (T * k,)).cpu().numpy()
    assert np.array_equal(ginv, inv)
    rtok = run.inter("row_token", torch.int32, (R,)).cpu().numpy()
    assert np.array_equal(rtok[inv], np.arange(T * k) // k)
    pad = np.ones(R, dtype=bool)
    pad[inv] = False
    pad[offsets[-1]:] = False                      # rows past the last expert are never written
    assert np.all(rtok[pad] == -1)
    # every assignment row of y and of its sum of squares (padding rows excluded)
    sel = torch.as_tensor(ginv.astype(np.int64), device=run.out.device)
    y = host(run.inter("y", act, (R, L))[sel]).reshape(T, k, L)
    y_ref = ref.pop("y")
    res["y"], _ = assert_close_stored(y, y_ref, f"{w.name} y (all {T * k} rows)", rel=rel, stored_bits=bits)
    del y
    ss = run.inter("ss", torch.float32, (R, L // 32))[sel].double().sum(1).cpu().numpy().reshape(T, k)
    ss_ref = ref.pop("ss")
    if oracle_modes.get("norm_mode") == "input_scaled":
        # the input-scaled norm takes the squares of u = y * (1 + gain): the CUDA path's
        # partials are of u, the oracle's stored sums of y
        gam = host(inp["gamma"])
        gam = gam[gidx] if gam.ndim == 2 else gam
        ss_ref = np.sum((y_ref * (1.0 + gam)) ** 2, axis=-1)
    del y_ref
    res["ss"], _ = assert_close(ss, ss_ref, f"{w.name} sum of squares", rel=2 * rel)
    res["act_adopted"] = ref.get("act_adopted", 0)
    return res


def expected_permutation(idx: np.ndarray, E: int):
    """Integer definition of the expert-ordered rows: assignments a = t*k + j grouped by
    expert, ascending a inside each expert, each expert's group padded to 16 rows."""
    flat = idx.reshape(-1)
    counts = np.bincount(flat, minlength=E)
    padded = (counts + 15) // 16 * 16
    offsets = np.concatenate([[0], np.cumsum(padded)])
    inv = np.empty(flat.size, dtype=np.int64)
    for e in range(E):
        a = np.nonzero(flat == e)[0]
        inv[a] = offsets[e] + np.arange(a.size)
    return counts, offsets, inv
