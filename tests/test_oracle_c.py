"""Pins of the plain-C FP64 reference (oracle/latent_moe_ref.c), on the CPU.

The C reference is checked through its whole-block entry point only: tiny blocks are built
whose structure makes a printed example of the pages, a closed form or a brute-force answer
come out of the full forward (identity pooler / unpooler, experts whose output direction is
fixed by construction, router rows that produce chosen logits). It is also compared with the
numpy oracle -- an independent implementation of the same definition -- on seeded inputs in
every mode both support.
"""
import ctypes
import functools
import itertools
import math

import numpy as np
import pytest

import oracle
import workloads as W
from golden_io import floats, lines
from oracle import cref


@pytest.fixture(scope="module", autouse=True)
def built():
    cref.build()


def silu(a):
    return a / (1.0 + math.exp(-a))


def block(x, W_router, W_pool, Wg, Wu, Wd, gamma, W_unpool, k, eps, **kw):
    return cref.latent_moe_forward_c(np.asarray(x, float), np.asarray(W_router, float), np.asarray(W_pool, float),
                                     (np.asarray(Wg, float), np.asarray(Wu, float), np.asarray(Wd, float)),
                                     np.asarray(gamma, float), np.asarray(W_unpool, float), k, eps, **kw)


# ----------------------------------------------------------------- printed examples
def norm_rows():
    for s in lines("norm_examples.txt"):
        name, v, w, centred, scaled, dec = [p.strip() for p in s.split("|")]
        yield name, floats(v), floats(w), floats(centred), floats(scaled), int(dec)


@pytest.mark.parametrize("row", list(norm_rows()), ids=lambda r: r[0])
@pytest.mark.parametrize("mode", ["centred", "input_scaled"])
def test_per_expert_norm_examples_through_the_whole_block(row, mode):
    """One expert, k = 1 (weight 1), identity pooler and unpooler, eps = 0. With z = x = (1, 1)
    and gate = up = identity, h = silu(1) (1, 1), so W_down = diag(v) makes the expert output
    silu(1) v: the block returns the per-expert norm of v with gain 1 + w (scale-invariant)."""
    name, v, w, centred, scaled, dec = row
    I2 = np.eye(2)
    out = block([[1.0, 1.0]], np.zeros((1, 2)), I2, I2[None], I2[None], np.diag(v)[None], np.array([w]), I2, 1,
                0.0, norm_mode=mode)
    want = centred if mode == "centred" else scaled
    # one unit in the last printed place: the page rounds an intermediate (4.301) before dividing
    assert np.allclose(out["out"][0], want, rtol=0, atol=10.0 ** -dec + 1e-12), (out["out"][0], want)
    assert out["g"][0, 0] == 1.0


def test_norm_before_mix_counter_example_through_the_whole_block():
    """Two experts, k = 2, equal router logits (weights 1/2 each), eps = 0, gain 1: expert 0's
    output lies on the first axis, expert 1's on the second, with the printed magnitudes 10
    and 1. Each is normalised before the weighted sum, so the block returns the printed
    per-expert result, not the printed normalise-after-mixing one."""
    rows = {s.split()[0]: floats(" ".join(s.split()[1:])) for s in lines("norm_before_mix.txt") if
            not s.startswith("output")}
    outs = [floats(" ".join(s.split()[1:])) for s in lines("norm_before_mix.txt") if s.startswith("output")]
    I2 = np.eye(2)
    # x = (1, 1): expert 0 sees a = u = (2, 0), expert 1 a = u = (0, 2), so h = 2 silu(2) e_i
    Wg = np.array([[[1, 1], [0, 0]], [[0, 0], [1, 1]]], float)
    scale = 2.0 * silu(2.0) * 2.0
    Wd = np.array([np.diag([outs[0][0] / scale * 2, 1.0]), np.diag([1.0, outs[1][1] / scale * 2])])
    out = block([[1.0, 1.0]], np.zeros((2, 2)), I2, Wg, Wg, Wd, np.zeros((2, 2)), I2, 2, 0.0)
    assert np.allclose(out["g"][0], rows["weights"], atol=1e-15)
    assert list(out["idx"][0]) == [0, 1]               # equal keys: lower index first
    assert np.allclose(out["out"][0], rows["per_expert_then_mix"], atol=1e-12)
    assert not np.allclose(out["out"][0], rows["mix_then_normalise"], atol=1e-2)


def test_router_renormalisation_example_in_sigmoid_mode():
    """Eight experts, k = 8, sigmoid scores chosen through the router rows (x = 1, logit =
    ln(s / (1 - s))): the weights are the printed renormalised scores."""
    rows = {s.split()[0]: floats(" ".join(s.split()[1:])) for s in lines("router_examples.txt")
            if s.split()[0] in ("scores", "weights")}
    s = np.array(rows["scores"])
    Wr = np.log(s / (1 - s))[:, None]
    E, D = 8, 1
    out = block([[1.0]], Wr, np.ones((1, 1)), np.ones((E, 1, 1)), np.ones((E, 1, 1)), np.ones((E, 1, 1)),
                np.zeros((E, 1)), np.ones((1, 1)), 8, 1e-6, router_mode="sigmoid")
    assert list(out["idx"][0]) == list(range(8))       # scores are printed in descending order
    assert np.allclose(out["g"][0], rows["weights"], atol=0.005)
    assert abs(out["g"][0].sum() - 1.0) < 1e-12


def test_router_bias_example_selects_but_does_not_weight():
    """The printed bias case: with logit multiplier 1/sqrt(32), expert 17 (logit 2.77, bias
    -0.30, key 0.32) loses the last of 8 slots to expert 90 (logit -2.29, bias +0.03, key
    0.43); the weights still come from the unbiased scores."""
    cases = {int(s.split()[1]): floats(" ".join(s.split()[2:])) for s in lines("router_examples.txt")
             if s.startswith("bias_case")}
    E, k = 91, 8
    scale = 1.0 / math.sqrt(32.0)
    logits = np.zeros(E)
    bias = np.full(E, -1.0)
    logits[:7] = 12.0                                  # seven clear winners (s ~ 0.89)
    bias[:7] = 0.0
    for e, (logit, _, s_printed, b, key_printed) in cases.items():
        logits[e] = logit
        bias[e] = b
        s = 1.0 / (1.0 + math.exp(-scale * logit))
        assert abs(s - s_printed) < 0.005 and abs(s + b - key_printed) < 0.005
    out = block([[1.0]], logits[:, None], np.ones((1, 1)), np.ones((E, 1, 1)), np.ones((E, 1, 1)),
                np.ones((E, 1, 1)), np.zeros((E, 1)), np.ones((1, 1)), k, 1e-6, router_mode="sigmoid",
                logit_scale=scale, router_bias=bias)
    sel = list(out["idx"][0])
    assert 90 in sel and 17 not in sel and sel[-1] == 90
    s = 1.0 / (1.0 + np.exp(-scale * logits[sel]))
    assert np.allclose(out["g"][0], s / (s.sum() + 1e-15), rtol=1e-14)


# ------------------------------------------------------------ brute force, closed forms
@pytest.mark.parametrize("seed", range(6))
def test_top_k_equals_brute_force_over_all_subsets_with_ties(seed):
    rng = np.random.default_rng(seed)
    E, k, D = 8, 3, 4
    Wr = rng.standard_normal((E, D))
    Wr[5] = Wr[2]                                      # exact ties: the lower index must win
    Wr[7] = Wr[1]
    x = rng.standard_normal((5, D))
    out = block(x, Wr, np.eye(D), np.ones((E, D, D)), np.ones((E, D, D)), np.ones((E, D, D)),
                np.zeros((E, D)), np.eye(D), k, 1e-6)
    for t in range(x.shape[0]):
        key = Wr @ x[t]
        # largest sum of keys; among equal sums the lexicographically smallest index set
        best = max(itertools.combinations(range(E), k), key=lambda c: (sum(key[list(c)]), [-i for i in c]))
        assert sorted(out["idx"][t]) == sorted(best), (t, out["idx"][t], best)
        ks = key[out["idx"][t]]
        assert all(ks[i] >= ks[i + 1] for i in range(k - 1))  # key descending
        assert abs(out["g"][t].sum() - 1.0) < 1e-12


def test_k_one_gives_weight_exactly_one():
    w = W.WORKLOADS["tiny"]
    inp = W.make_inputs(w, "cpu")
    out = cref.latent_moe_forward_c(inp["x"], inp["W_router"], inp["W_pool"],
                                    (inp["W_gate"], inp["W_up"], inp["W_down"]), inp["gamma"], inp["W_unpool"], 1,
                                    w.eps)
    assert np.all(out["g"] == 1.0)


def test_k_equals_E_with_identical_experts_is_one_dense_expert():
    """All experts and gains equal and k = E: the weights sum to 1, so the block is the
    unpooler of one normalised dense expert on the pooled token."""
    rng = np.random.default_rng(3)
    T, D, L, I, E = 5, 12, 8, 6, 4
    x = rng.standard_normal((T, D))
    Wr = rng.standard_normal((E, D))
    Wp = rng.standard_normal((L, D)) / math.sqrt(D)
    Wg1, Wu1, Wd1 = rng.standard_normal((I, L)), rng.standard_normal((I, L)), rng.standard_normal((L, I))
    g1 = 0.3 * rng.standard_normal(L)
    Wun = rng.standard_normal((D, L))
    out = block(x, Wr, Wp, np.repeat(Wg1[None], E, 0), np.repeat(Wu1[None], E, 0), np.repeat(Wd1[None], E, 0),
                np.repeat(g1[None], E, 0), Wun, E, 1e-6)
    dense = oracle.unpooler(oracle.centred_rmsnorm(oracle.expert_ffn(oracle.pooler(x, Wp), Wg1, Wu1, Wd1), g1, 1e-6),
                            Wun)
    assert np.allclose(out["out"], dense, rtol=1e-12, atol=1e-12)


def test_token_permutation_permutes_the_outputs_exactly():
    w = W.WORKLOADS["tiny"]
    inp = W.make_inputs(w, "cpu")
    perm = np.random.default_rng(1).permutation(w.T)
    ex = (inp["W_gate"], inp["W_up"], inp["W_down"])
    a = cref.latent_moe_forward_c(inp["x"], inp["W_router"], inp["W_pool"], ex, inp["gamma"], inp["W_unpool"], w.k,
                                  w.eps)
    b = cref.latent_moe_forward_c(inp["x"][perm], inp["W_router"], inp["W_pool"], ex, inp["gamma"], inp["W_unpool"],
                                  w.k, w.eps)
    assert np.array_equal(a["out"][perm], b["out"]) and np.array_equal(a["idx"][perm], b["idx"])


# ------------------------------------------------------------ the two implementations
MODES = [
    dict(),
    dict(router_mode="sigmoid", logit_scale=1.0 / math.sqrt(32.0), routed_scaling=1.0, bias=True),
    dict(norm_mode="input_scaled", shared_gamma=True),
    dict(pre_norm=True),
    dict(router_mode="sigmoid", logit_scale=0.5, routed_scaling=2.5, norm_mode="input_scaled", pre_norm=True),
]


AGREE = {
    "tiny": W.WORKLOADS["tiny"],
    # the mid workload's expert count, top-k and dtype at a width that generates quickly
    "mid_narrow": W.Workload("mid_narrow", T=24, D=512, L=256, I=384, E=64, k=4, dtype="bf16", seed=2),
}


@functools.lru_cache(maxsize=None)
def agree_inputs(name):
    return W.make_inputs(AGREE[name], "cpu")


@pytest.mark.parametrize("name,T", [("tiny", 16), ("mid_narrow", 24)])
@pytest.mark.parametrize("mode", range(len(MODES)))
def test_c_reference_agrees_with_the_numpy_oracle(name, T, mode):
    m = dict(MODES[mode])
    w = AGREE[name]
    inp = agree_inputs(name)
    f = oracle.as_f64
    rng = np.random.default_rng(mode)
    bias = 0.05 * rng.standard_normal(w.E) if m.pop("bias", False) else None
    gamma = f(inp["gamma"])[0] if m.pop("shared_gamma", False) else f(inp["gamma"])
    pre = 0.3 * rng.standard_normal(w.L) if m.pop("pre_norm", False) else None
    x = f(inp["x"])[:T]
    ex = (f(inp["W_gate"]), f(inp["W_up"]), f(inp["W_down"]))
    c = cref.latent_moe_forward_c(x, f(inp["W_router"]), f(inp["W_pool"]), ex, gamma, f(inp["W_unpool"]), w.k, w.eps,
                                  router_bias=bias, pre_norm_gain=pre, **m)
    kw = {("router_bias" if k == "bias" else k): v for k, v in m.items()}
    r = oracle.latent_moe_forward(x, f(inp["W_router"]), f(inp["W_pool"]), ex, gamma, f(inp["W_unpool"]), w.k, w.eps,
                                  router_bias=bias, pre_norm_gain=pre, **kw)
    assert np.array_equal(c["idx"], r["idx"])
    assert np.allclose(c["g"], r["g"], rtol=1e-13, atol=1e-15)
    scale = np.abs(r["out"]).max()
    assert np.abs(c["out"] - r["out"]).max() <= 1e-12 * scale


# ------------------------------------------------------------------- NVFP4 experts
def test_c_decoders_match_the_ocp_tables_and_every_e4m3_byte():
    """The C decoders of the 4-bit E2M1 values and the E4M3 block-scale bytes against the
    OCP MX v1.0 tables (golden files) and, for E4M3, every byte against torch's float8."""
    for s in lines("fp4_e2m1.txt"):
        code, val = s.split()
        got = cref.e2m1_value(int(code))
        assert got == float(val) and math.copysign(1.0, got) == (-1.0 if val.startswith("-") else 1.0)
    for s in lines("fp8_e4m3.txt"):
        b, val = s.split()
        got = cref.e4m3_value(int(b, 16))
        assert (math.isnan(got) and val == "nan") or got == float(val)
    import torch
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([cref.e4m3_value(b) for b in range(256)])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(got[~np.isnan(got)], ref[~np.isnan(ref)])


NVFP4_AGREE = [
    W.Workload("c_nvfp4_tiny", T=12, D=256, L=128, I=128, E=8, k=2, dtype="bf16", seed=4, experts="nvfp4"),
    # the NVFP4 parity workloads' expert count and top-k at a narrow width
    W.Workload("c_nvfp4_mid", T=10, D=512, L=256, I=384, E=64, k=4, dtype="bf16", seed=9, experts="nvfp4"),
]


@pytest.mark.parametrize("w", NVFP4_AGREE, ids=lambda w: w.name)
@pytest.mark.parametrize("mode", [0, 2])
def test_c_reference_with_nvfp4_experts_agrees_with_the_numpy_oracle(w, mode):
    """The C block decoding NVFP4 codes itself against the numpy oracle on the dequantised
    weights (the same codes): routing identical, outputs to 1e-12 of their scale."""
    m = dict(MODES[mode])
    inp = W.make_inputs(w, "cpu")
    f = oracle.as_f64
    gamma = f(inp["gamma"])[0] if m.pop("shared_gamma", False) else f(inp["gamma"])
    q = [(inp[n + "_codes"], inp[n + "_scales"], inp[n + "_mscale"]) for n in ("W_gate", "W_up", "W_down")]
    c = cref.latent_moe_forward_c(inp["x"], inp["W_router"], inp["W_pool"], q, gamma, inp["W_unpool"], w.k, w.eps,
                                  nvfp4=True, **m)

    def deq(e):
        return tuple(oracle.dequantize_nvfp4(cd[e].numpy(), sc[e].numpy(), float(ms[e])) for cd, sc, ms in q)
    r = oracle.latent_moe_forward(f(inp["x"]), f(inp["W_router"]), f(inp["W_pool"]), deq, gamma, f(inp["W_unpool"]),
                                  w.k, w.eps, **m)
    assert np.array_equal(c["idx"], r["idx"])
    assert np.abs(c["out"] - r["out"]).max() <= 1e-12 * np.abs(r["out"]).max()


def test_c_reference_rejects_nvfp4_widths_that_are_not_whole_blocks():
    w = NVFP4_AGREE[0]
    inp = W.make_inputs(w, "cpu")
    q = [(inp[n + "_codes"], inp[n + "_scales"], inp[n + "_mscale"]) for n in ("W_gate", "W_up", "W_down")]
    c = cref.RefCfg(T=1, D=w.D, L=120, I=w.I, E=w.E, k=w.k, eps=w.eps)
    mats = [cref.RefNvfp4(0, 0, 0) for _ in range(3)]
    out = np.zeros((1, w.D))
    rc = cref.lib().ref_latent_moe_forward_nvfp4(ctypes.byref(c), 0, 0, 0, *[ctypes.addressof(m) for m in mats], 0, 0,
                                                 out.ctypes.data, 0, 0)
    assert rc == -1
