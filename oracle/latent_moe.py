"""FP64 oracle of the latent mixture-of-experts block of Muse Spark Open.

TEST INFRASTRUCTURE. This module is the plain definition the CUDA library is checked
against; it is never on the product path. Only tests/, __graft_entry__.smoke() and
bench.py (its cpu_baseline / reference leg) may import it.

Every input is taken exactly as stored (bfloat16 / float32 values widened to float64)
and nothing is rounded in between. Library primitives used as steps: numpy matmul
(float64), numpy exp / sqrt, numpy lexsort. No blocking or fusion beyond the
definition; the only reordering is that (token, slot) pairs are grouped by expert
before the expert FFN runs ("dispatch"), which does not change any per-token value.

Sources (page title, then section / equation):
  * "Muse Spark Open deep dive" (gangliao.me), §4.2 router, §4.3 pool -> compute ->
    unpool with the block equation y = W_up_proj sum_i g_i N_post(E_i(z)),
    §4.4 norms inside the MoE, §5.3 RMSNorm variants table and worked example;
  * "Muse Spark Open: Normerhaltende Gates sind keine Normgarantie" (flozi.net),
    "Zwei Normierungsreihenfolgen" (C_gamma / I_gamma and the (1,1), diag(2,1)
    example) and "Latente Experts: Normierung vor der gewichteten Summe";
  * the block as fixed for this library: softmax over all E logits, top-k with ties to
    the lower index, weights renormalised over the selected set, a zero-centred-gain
    RMSNorm y/rms(y)*(1+gamma_e) per expert.

Readings where the pages are open or disagree:
  * router score: softmax (default); the pages' released router (sigmoid of the logit
    times 1/sqrt(32), selection-only bias, s/(sum s + 1e-15) * routed_scaling_factor)
    is `router_mode="sigmoid"`;
  * order of the k selected experts: key descending, ties to the lower index; this is
    the "routing order" the combine sums in;
  * per-expert output norm: centred form with a per-expert gain (default); the pages'
    shared input-scaled form is `norm_mode="input_scaled"`;
  * no pre-expert norm unless `pre_norm_gain` is given (pages: centred, eps 1e-5);
  * the feed-forward sublayer around the block (pre-norm, post-norm, residual gate;
    deep dive §2.1 steps 6-7, §5.2, §5.3) only when its parameters are given; gains are
    used as 1 + w exactly (the pages' ports round 1 + w to bfloat16 first).

Parity pins (tests/test_oracle_pins.py): every function here is pinned by a worked
example printed on the pages, a closed form, a brute-force enumeration or an
invariant; none is marked "parity unpinned".
"""
from __future__ import annotations

import itertools
from typing import Callable, Dict, List, Optional, Sequence, Tuple, Union

import numpy as np

__all__ = [
    "router_logits", "select_topk", "softmax_weights", "sigmoid_weights", "route",
    "topk_alternatives", "pooler", "silu", "expert_ffn", "centred_rmsnorm",
    "input_scaled_rmsnorm", "combine", "unpooler", "latent_moe_forward", "as_f64",
    "moe_flops_per_token", "expert_param_count", "residual_gate_coefficients", "residual_gate",
    "round_bf16", "nvfp4_activation",
]

Array = np.ndarray
ExpertSource = Union[Tuple[Array, Array, Array], Callable[[int], Tuple[Array, Array, Array]]]


def as_f64(t) -> Array:
    """Widen a stored tensor (torch bf16/f32 or numpy) to float64, exactly."""
    try:
        import torch
        if isinstance(t, torch.Tensor):
            return t.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(t, dtype=np.float64)


# ---------------------------------------------------------------------------------------
# (a1) router logits -- deep dive §4.2 step 1: l = W_r h on the full-width hidden state
# ---------------------------------------------------------------------------------------
def router_logits(x: Array, W_router: Array) -> Array:
    """l[t, e] = sum_d W_router[e, d] * x[t, d]; x [T, D], W_router [E, D] -> [T, E]."""
    return x @ W_router.T


# ---------------------------------------------------------------------------------------
# (a2) selection and weights -- deep dive §4.2 steps 3-5 and the routing equation
# ---------------------------------------------------------------------------------------
def select_topk(keys: Array, k: int) -> Array:
    """Indices of the k largest keys per row, ordered by (key desc, index asc)."""
    T, E = keys.shape
    index = np.broadcast_to(np.arange(E), (T, E))
    order = np.lexsort((index, -keys), axis=-1)   # primary -key, secondary index
    return order[:, :k].astype(np.int64)


def softmax_weights(logits: Array, idx: Array) -> Array:
    """Softmax over all E logits, renormalised on the selected set.

    softmax(l)_j / sum_{j' in S} softmax(l)_{j'} = exp(l_j - m) / sum_{S} exp(l - m)
    with m the largest selected logit (the full-softmax denominator cancels).
    """
    sel = np.take_along_axis(logits, idx, axis=-1)
    m = sel.max(axis=-1, keepdims=True)
    p = np.exp(sel - m)
    return p / p.sum(axis=-1, keepdims=True)


def sigmoid_weights(logits: Array, idx: Array, logit_scale: float, routed_scaling: float = 1.0,
                    renorm_eps: float = 1e-15) -> Array:
    """Released Muse Spark router weights (deep dive §4.2 step 5; Norm gates page):
    g_i = routed_scaling * s_i / (sum_{j in T} s_j + 1e-15), s = sigmoid(scale * l),
    computed from the unbiased scores."""
    s = _sigmoid(logit_scale * np.take_along_axis(logits, idx, axis=-1))
    return routed_scaling * s / (s.sum(axis=-1, keepdims=True) + renorm_eps)


def _sigmoid(a: Array) -> Array:
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-a))


def route(logits: Array, k: int, bias: Optional[Array] = None, router_mode: str = "softmax",
          logit_scale: float = 1.0, routed_scaling: float = 1.0) -> Tuple[Array, Array, Array]:
    """Returns (idx [T,k], g [T,k], keys [T,E]).

    softmax mode: key = l + b; g = softmax over the selected (unbiased) logits.
    sigmoid mode (pages): s = sigmoid(scale*l); key = s + b; g = s/(sum s + 1e-15)*rsf.
    The bias only changes which experts are selected (deep dive §4.2 step 4-5).
    """
    b = 0.0 if bias is None else np.asarray(bias, dtype=np.float64)[None, :]
    if router_mode == "softmax":
        keys = logits + b
        idx = select_topk(keys, k)
        g = softmax_weights(logits, idx)
    elif router_mode == "sigmoid":
        keys = _sigmoid(logit_scale * logits) + b
        idx = select_topk(keys, k)
        g = sigmoid_weights(logits, idx, logit_scale, routed_scaling)
    else:
        raise ValueError(router_mode)
    return idx, g, keys


def topk_alternatives(keys_row: Array, k: int, tol: float) -> List[Tuple[int, ...]]:
    """All index sets that are a valid top-k of one row when keys within `tol` of the
    k-th largest key are treated as tied. Used where several routings are correct: a
    set outside this list is wrong. Each set is returned sorted ascending."""
    order = select_topk(keys_row[None, :], keys_row.shape[0])[0]
    kth = keys_row[order[k - 1]]
    sure = [int(e) for e in order if keys_row[e] > kth + tol]
    near = [int(e) for e in order if abs(keys_row[e] - kth) <= tol]
    need = k - len(sure)
    return [tuple(sorted(sure + list(c))) for c in itertools.combinations(near, need)]


# ---------------------------------------------------------------------------------------
# (a4) pooler and (a10) unpooler -- deep dive §4.3 steps 1 and 7 (bias-free linear)
# ---------------------------------------------------------------------------------------
def pooler(x: Array, W_pool: Array) -> Array:
    """z = W_pool x per token; W_pool [L, D] stored [out, in]."""
    return x @ W_pool.T


def unpooler(c: Array, W_unpool: Array) -> Array:
    """out = W_unpool c per token; W_unpool [D, L] stored [out, in]."""
    return c @ W_unpool.T


# ---------------------------------------------------------------------------------------
# (a6, a7) expert SwiGLU -- deep dive §4.3 step 4: E_i(z) = W_down(SiLU(W_gate z) * W_up z)
# ---------------------------------------------------------------------------------------
def silu(a: Array) -> Array:
    """SiLU(a) = a * sigmoid(a)."""
    return a * _sigmoid(a)


def expert_ffn(z: Array, W_gate: Array, W_up: Array, W_down: Array,
               act: Optional[Callable[[Array], Array]] = None) -> Array:
    """Rows of z [n, L] through one expert; W_gate/W_up [I, L], W_down [L, I]. act, when
    given, maps each GEMM's activation operand (z, then the SwiGLU output h) to the values
    the GEMM multiplies (the W4A4 mode's quantise-dequantise)."""
    if act is not None:
        z = act(z, 0)
    a = z @ W_gate.T
    u = z @ W_up.T
    h = silu(a) * u
    if act is not None:
        h = act(h, 1)
    return h @ W_down.T


def nvfp4_activation(v: Array, ref=None, adopted=None) -> Array:
    """W4A4 operand of an expert GEMM: the activation as the kernels store it (bfloat16),
    quantised per 16 to E2M1 codes with E4M3 scales, and dequantised (oracle.nvfp4); ref /
    adopted as in quantize_activations_nvfp4."""
    from .nvfp4 import dequantize_activations_nvfp4, quantize_activations_nvfp4
    codes, scales = quantize_activations_nvfp4(round_bf16(v), ref=ref, adopted=adopted)
    return dequantize_activations_nvfp4(codes, scales)


# ---------------------------------------------------------------------------------------
# (a8) per-expert RMSNorm -- Norm gates page, C_gamma and I_gamma; deep dive §4.4, §5.3
# ---------------------------------------------------------------------------------------
def centred_rmsnorm(v: Array, gain_offset: Array, eps: float) -> Array:
    """Output-scaled ("centred") form: v / sqrt(mean(v^2) + eps) * (1 + w)."""
    r = np.sqrt(np.mean(v * v, axis=-1, keepdims=True) + eps)
    return v / r * (1.0 + gain_offset)


def input_scaled_rmsnorm(v: Array, gain_offset: Array, eps: float) -> Array:
    """Input-scaled form: u / sqrt(mean(u^2) + eps) with u = v * (1 + w)."""
    u = v * (1.0 + gain_offset)
    r = np.sqrt(np.mean(u * u, axis=-1, keepdims=True) + eps)
    return u / r


# ---------------------------------------------------------------------------------------
# (a9) weighted combine -- deep dive §4.3 step 6; weights applied after each norm
# ---------------------------------------------------------------------------------------
def combine(n: Array, g: Array) -> Array:
    """c[t] = sum_j g[t, j] * n[t, j]; n [T, k, L], g [T, k]; j summed in routing order."""
    c = np.zeros((n.shape[0], n.shape[2]))
    for j in range(n.shape[1]):
        c = c + g[:, j:j + 1] * n[:, j, :]
    return c


# ---------------------------------------------------------------------------------------
# the feed-forward sublayer around the block -- deep dive §2.1 steps 6-7 and §5.3 norm
# table (pre_feedforward_layernorm: centred, eps 1e-5; post_feedforward_layernorm:
# scale first, then normalise, eps 1e-8), §5.2 norm-preserving residual gate
# ---------------------------------------------------------------------------------------
def round_bf16(a: Array) -> Array:
    """Round float64 values to the nearest bfloat16 (8 significant bits, ties to even),
    returned as float64. Used where the pages' implementation stores an activation in
    bfloat16 before a decision is taken on it."""
    m, e = np.frexp(np.asarray(a, dtype=np.float64))
    return np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)


def residual_gate_coefficients(gate: Array, temperature: float = 0.3, floor: float = 1e-3):
    """Per-channel (alpha, beta) of the residual gate with parameters g:
    beta = sigmoid(g / T) weights the branch, alpha = sqrt(max(sigmoid(-g / T) * (1 + beta),
    floor)) the residual stream; where the floor is inactive alpha^2 = 1 - beta^2."""
    w = gate / temperature
    beta = _sigmoid(w)
    alpha = np.sqrt(np.maximum(_sigmoid(-w) * (1.0 + beta), floor))
    return alpha, beta


def residual_gate(x: Array, f: Array, gate: Array, temperature: float = 0.3, floor: float = 1e-3) -> Array:
    """alpha * x + beta * f per channel: x the residual stream, f the normalised branch."""
    alpha, beta = residual_gate_coefficients(gate, temperature, floor)
    return alpha * x + beta * f


# ---------------------------------------------------------------------------------------
# the whole block
# ---------------------------------------------------------------------------------------
def latent_moe_forward(x: Array, W_router: Array, W_pool: Array, experts: ExpertSource,
                       gamma: Array, W_unpool: Array, k: int, eps: float,
                       router_bias: Optional[Array] = None, router_mode: str = "softmax",
                       logit_scale: float = 1.0, routed_scaling: float = 1.0,
                       norm_mode: str = "centred", pre_norm_gain: Optional[Array] = None,
                       pre_norm_eps: float = 1e-5, routing: Optional[Tuple[Array, Array]] = None,
                       ffn_pre_gain: Optional[Array] = None, ffn_pre_eps: float = 1e-5,
                       ffn_post_gain: Optional[Array] = None, ffn_post_eps: float = 1e-8,
                       gate: Optional[Array] = None, gate_temperature: float = 0.3, gate_floor: float = 1e-3,
                       xn_round: Optional[str] = None, act_format: str = "bf16",
                       act_ref: Optional[Callable] = None) -> Dict[str, Array]:
    """Forward pass of the latent-MoE block for every row of x, in float64.

    experts: (W_gate [E,I,L], W_up [E,I,L], W_down [E,L,I]) or a callable e -> the three
    [out, in] matrices of expert e (so full-size weights need not sit in host memory).
    gamma: [E, L] per-expert gain offsets, or [L] for one shared gain.
    routing: optional (idx, g) from one of this oracle's own alternative routings.
    ffn_pre_gain / ffn_post_gain / gate: the feed-forward sublayer's pre-norm, post-norm
    and residual gate around the block; x is then the residual stream and out its next
    value: xn = centred(x), f = block(xn), fn = input-scaled(f), out = alpha x + beta fn.
    xn_round="bf16" rounds xn to bfloat16 before the router and the pooler read it, as the
    pages' implementation stores it (the routing decision is then taken on the same values
    the bfloat16 kernels see). act_format="nvfp4" runs the expert GEMMs W4A4: their
    activation operands (z rows, SwiGLU outputs) go through nvfp4_activation. act_ref, for
    W4A4: a callable (token rows, slots) -> ((z codes, z scales), (h codes, h scales)) of
    those assignments from another implementation, whose decisions are adopted where they
    sit at a rounding boundary (quantize_activations_nvfp4); "act_adopted" counts them.

    Returns every intermediate: xn, logits, keys, idx, g, z, y [T,k,L], ss [T,k], n, c,
    f (the block's output), out.
    """
    T = x.shape[0]
    x_res = x
    if ffn_pre_gain is not None:
        x = centred_rmsnorm(x, ffn_pre_gain, ffn_pre_eps)
        if xn_round == "bf16":
            x = round_bf16(x)
    xn = x
    logits = router_logits(x, W_router)                                  # (a1)
    idx, g, keys = route(logits, k, router_bias, router_mode, logit_scale, routed_scaling)
    if routing is not None:
        idx, g = routing
    z = pooler(x, W_pool)                                                # (a4)
    if pre_norm_gain is not None:
        z = centred_rmsnorm(z, pre_norm_gain, pre_norm_eps)
    L = z.shape[1]
    y = np.zeros((T, k, L))
    get = experts if callable(experts) else (lambda e: (experts[0][e], experts[1][e], experts[2][e]))
    adopted = [0]
    for e in np.unique(idx):                                             # (a3) dispatch
        tok, slot = np.nonzero(idx == e)
        Wg, Wu, Wd = get(int(e))
        act = None
        if act_format == "nvfp4":
            refs = act_ref(tok, slot) if act_ref is not None else (None, None)
            act = (lambda v, stage, refs=refs: nvfp4_activation(v, refs[stage], adopted))
        y[tok, slot, :] = expert_ffn(z[tok], as_f64(Wg), as_f64(Wu), as_f64(Wd), act)  # (a6, a7)
    gam = gamma[idx] if gamma.ndim == 2 else np.broadcast_to(gamma, (T, k, L))
    if norm_mode == "centred":                                           # (a8)
        n = centred_rmsnorm(y, gam, eps)
    elif norm_mode == "input_scaled":
        n = input_scaled_rmsnorm(y, gam, eps)
    else:
        raise ValueError(norm_mode)
    c = combine(n, g)                                                    # (a9)
    f = unpooler(c, W_unpool)                                            # (a10)
    ss = np.sum(y * y, axis=-1)
    out = f if ffn_post_gain is None else input_scaled_rmsnorm(f, ffn_post_gain, ffn_post_eps)
    if gate is not None:
        out = residual_gate(x_res, out, gate, gate_temperature, gate_floor)
    return {"xn": xn, "logits": logits, "keys": keys, "idx": idx, "g": g, "z": z, "y": y, "ss": ss,
            "n": n, "c": c, "f": f, "out": out, "act_adopted": adopted[0]}


# ---------------------------------------------------------------------------------------
# accounting (deep dive §4.1 table and §4.3 comparison table)
# ---------------------------------------------------------------------------------------
def expert_param_count(L: int, I: int) -> int:
    """Parameters of one SwiGLU expert: gate and up [I, L], down [L, I]."""
    return 3 * L * I


def moe_flops_per_token(D: int, L: int, I: int, E: int, k: int) -> int:
    """Algorithmic multiply-add FLOPs of one token through the block: router, pooler,
    k experts, unpooler (2 per multiply-add; the norms' O(L) work is not counted)."""
    return 2 * (E * D + L * D + k * expert_param_count(L, I) + D * L)
