"""Pins of the FP64 oracle to things other than itself (CPU only).

Each test checks the oracle against a value printed on the pages (fixtures under
tests/golden/, each citing its page and section), a closed form, a brute-force
enumeration, or an invariant of the mathematics -- chosen so that a dropped term, a
wrong sign, a swapped operand or a transposed weight fails at least one of them.
"""
import itertools
import math

import numpy as np
import pytest

import oracle
from golden_io import floats, lines

RNG = np.random.default_rng(1234)


# ------------------------------------------------------------------ RMSNorm forms (a8)
def _norm_rows():
    for s in lines("norm_examples.txt"):
        name, v, w, cen, ins, dec = [p.strip() for p in s.split("|")]
        yield name, np.array(floats(v)), np.array(floats(w)), np.array(floats(cen)), \
            np.array(floats(ins)), int(dec)


@pytest.mark.parametrize("row", list(_norm_rows()), ids=lambda r: r[0])
def test_rmsnorm_worked_examples(row):
    name, v, w, cen, ins, dec = row
    # one unit in the last printed place: the deep dive prints 1/4.301 = 0.23250 as 0.233
    tol = 10.0 ** (-dec) + 1e-12
    np.testing.assert_allclose(oracle.centred_rmsnorm(v, w, 0.0), cen, rtol=0, atol=tol)
    np.testing.assert_allclose(oracle.input_scaled_rmsnorm(v, w, 0.0), ins, rtol=0, atol=tol)


def test_rmsnorm_rms_printed_in_deep_dive():
    rms = lambda a: math.sqrt(float(np.mean(a * a)))
    # deep dive §5.3 example also prints the RMS of both outputs: 1.92 and 1.00
    v, w = np.array([3.0, 1.0]), np.array([1.0, 0.0])
    assert abs(rms(oracle.centred_rmsnorm(v, w, 0.0)) - 1.92) < 0.005
    assert abs(rms(oracle.input_scaled_rmsnorm(v, w, 0.0)) - 1.00) < 0.005


@pytest.mark.parametrize("row", list(lines("norm_rms_examples.txt")))
def test_rmsnorm_epsilon_output_rms(row):
    eps, in_rms, out_rms, dec = floats(row)
    v = np.full(64, in_rms) * np.where(np.arange(64) % 2 == 0, 1.0, -1.0)
    got = oracle.centred_rmsnorm(v, np.zeros(64), eps)
    assert abs(math.sqrt(np.mean(got ** 2)) - out_rms) <= 0.5 * 10 ** (-int(dec))
    # closed form sqrt(ms/(ms+eps)) for any row
    y = RNG.normal(size=(5, 33)) * 1e-3
    ms = np.mean(y * y, axis=1)
    n = oracle.centred_rmsnorm(y, np.zeros(33), eps)
    np.testing.assert_allclose(np.sqrt(np.mean(n * n, axis=1)), np.sqrt(ms / (ms + eps)), rtol=1e-13)


def test_rmsnorm_unit_row_rms_equals_gain_rms():
    # all |y_i| equal: rms(N(y)) = rms(1+gamma) * sqrt(ms/(ms+eps))
    L, eps = 128, 1e-6
    gamma = RNG.normal(size=L) * math.sqrt(0.1)
    y = 0.37 * np.where(RNG.random(L) < 0.5, -1.0, 1.0)
    n = oracle.centred_rmsnorm(y, gamma, eps)
    expect = math.sqrt(np.mean((1 + gamma) ** 2)) * math.sqrt(0.37 ** 2 / (0.37 ** 2 + eps))
    assert abs(math.sqrt(np.mean(n * n)) - expect) < 1e-13


def test_input_scaled_norm_has_unit_rms_for_any_gain():
    v = RNG.normal(size=(4, 64))
    w = RNG.normal(size=64)
    n = oracle.input_scaled_rmsnorm(v, w, 0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(n * n, axis=1)), 1.0, rtol=1e-14)


def test_norm_is_scale_invariant_at_eps0():
    v = RNG.normal(size=(3, 40))
    g = RNG.normal(size=40) * 0.3
    np.testing.assert_allclose(oracle.centred_rmsnorm(7.5 * v, g, 0.0), oracle.centred_rmsnorm(v, g, 0.0),
                               rtol=1e-13)


# ------------------------------------------------------------------ combine (a9)
def test_norm_before_mix_counter_example():
    rows = {s.split()[0]: floats(" ".join(s.split()[1:])) for s in lines("norm_before_mix.txt")
            if not s.startswith("output")}
    outs = np.array([floats(" ".join(s.split()[1:])) for s in lines("norm_before_mix.txt")
                     if s.startswith("output")])
    w = np.array(rows["weights"])
    n = oracle.centred_rmsnorm(outs, np.zeros(2), 0.0)            # per expert
    c = oracle.combine(n[None], w[None])[0]
    np.testing.assert_allclose(c, rows["per_expert_then_mix"], rtol=1e-15)
    wrong = oracle.centred_rmsnorm(w @ outs, np.zeros(2), 0.0)
    np.testing.assert_allclose(wrong, rows["mix_then_normalise"], rtol=1e-15)
    assert np.abs(c - wrong).max() > 0.5


def test_combine_rms_bound_and_equality():
    # gamma = 0, eps = 0: every normalised row has RMS 1, weights sum to 1 => rms(c) <= 1,
    # equality iff all k rows are parallel.
    n = oracle.centred_rmsnorm(RNG.normal(size=(6, 4, 32)), np.zeros(32), 0.0)
    g = RNG.random((6, 4))
    g /= g.sum(1, keepdims=True)
    c = oracle.combine(n, g)
    assert np.all(np.sqrt(np.mean(c * c, axis=1)) <= 1.0 + 1e-14)
    same = np.repeat(n[:, :1], 4, axis=1)
    c2 = oracle.combine(same, g)
    np.testing.assert_allclose(np.sqrt(np.mean(c2 * c2, axis=1)), 1.0, rtol=1e-14)


def test_combine_weights_follow_slots():
    n = np.zeros((1, 3, 2))
    n[0, 0] = [1, 0]
    n[0, 1] = [0, 1]
    n[0, 2] = [1, 1]
    c = oracle.combine(n, np.array([[0.5, 0.3, 0.2]]))
    np.testing.assert_allclose(c[0], [0.7, 0.5], rtol=1e-15)


# ------------------------------------------------------------------ router (a1, a2)
def test_topk_brute_force_small():
    for E, k in [(8, 2), (16, 4), (9, 9), (12, 1)]:
        for _ in range(30):
            keys = RNG.normal(size=(1, E))
            idx = oracle.select_topk(keys, k)[0]
            best = max(itertools.combinations(range(E), k), key=lambda s: sum(keys[0, list(s)]))
            assert set(idx.tolist()) == set(best)
            # routing order: key descending
            assert np.all(np.diff(keys[0, idx]) <= 0)


def test_topk_ties_go_to_lower_index():
    keys = np.array([[0.5, 1.0, 0.5, 1.0, 0.5, 0.2]])
    assert oracle.select_topk(keys, 2)[0].tolist() == [1, 3]
    assert oracle.select_topk(keys, 3)[0].tolist() == [1, 3, 0]
    assert oracle.select_topk(keys, 5)[0].tolist() == [1, 3, 0, 2, 4]
    # brute force over ties: the lexicographically smallest index set among the maxima
    keys = np.round(RNG.normal(size=(1, 10)) * 2) / 2
    for k in range(1, 10):
        sel = oracle.select_topk(keys, k)[0]
        sets = list(itertools.combinations(range(10), k))
        vals = [sum(keys[0, list(s)]) for s in sets]
        best = max(vals)
        cands = sorted(tuple(sorted(s)) for s, v in zip(sets, vals) if abs(v - best) < 1e-12)
        # lower index wins each tie: the candidate with the smallest indices at equal keys
        ref = sorted(range(10), key=lambda e: (-keys[0, e], e))[:k]
        assert tuple(sorted(ref)) in cands
        assert sel.tolist() == ref


def test_softmax_weights_are_renormalised_full_softmax():
    logits = RNG.normal(size=(5, 16)) * 3
    idx = oracle.select_topk(logits, 4)
    g = oracle.softmax_weights(logits, idx)
    full = np.exp(logits) / np.exp(logits).sum(1, keepdims=True)
    sel = np.take_along_axis(full, idx, 1)
    np.testing.assert_allclose(g, sel / sel.sum(1, keepdims=True), rtol=1e-13)
    np.testing.assert_allclose(g.sum(1), 1.0, rtol=1e-15)
    # k = 1 gives weight exactly 1
    assert np.all(oracle.softmax_weights(logits, oracle.select_topk(logits, 1)) == 1.0)


def test_router_renormalisation_example():
    rows = {s.split()[0]: floats(" ".join(s.split()[1:])) for s in lines("router_examples.txt")
            if not s.startswith("bias_case")}
    s = np.array(rows["scores"])
    assert abs(s.sum() - 4.00) < 1e-12
    scale = 1 / math.sqrt(32)
    logits = np.log(s / (1 - s)) / scale                       # sigmoid^-1 of the scores
    g = oracle.sigmoid_weights(logits[None], np.arange(8)[None], scale, 1.0)[0]
    np.testing.assert_allclose(g, rows["weights"], atol=0.005 + 1e-12)
    assert abs(g.sum() - 1.0) < 1e-14


def test_router_selection_only_bias_example():
    cases = {int(s.split()[1]): floats(" ".join(s.split()[2:]))
             for s in lines("router_examples.txt") if s.startswith("bias_case")}
    E, k, scale = 256, 8, 1 / math.sqrt(32)
    logits = np.full(E, -20.0)
    winners = [3, 40, 77, 120, 150, 200, 250]
    logits[winners] = 12.0
    bias = np.zeros(E)
    for e, (logit, scaled, s_pr, b, key_pr) in cases.items():
        logits[e] = logit
        bias[e] = b
        s = 1 / (1 + math.exp(-scale * logit))
        assert abs(s - s_pr) < 0.005
        assert abs(s + b - key_pr) < 0.005
        if not math.isnan(scaled):
            assert abs(scale * logit - scaled) < 0.005
    idx, g, keys = oracle.route(logits[None], k, bias, "sigmoid", scale, 1.0)
    assert 90 in idx[0] and 17 not in idx[0]
    # the weight of expert 90 comes from its raw score, not from score + bias
    s_sel = 1 / (1 + np.exp(-scale * logits[idx[0]]))
    j = list(idx[0]).index(90)
    assert abs(g[0, j] - s_sel[j] / (s_sel.sum() + 1e-15)) < 1e-15
    assert abs(s_sel[j] - 0.40) < 0.005
    # without the bias, expert 17 would have taken the slot
    idx0, _, _ = oracle.route(logits[None], k, None, "sigmoid", scale, 1.0)
    assert 17 in idx0[0] and 90 not in idx0[0]


def test_softmax_mode_bias_selects_but_does_not_weight():
    logits = np.array([[1.0, 0.9, 0.0, -1.0]])
    bias = np.array([0.0, 0.0, 2.0, 0.0])
    idx, g, _ = oracle.route(logits, 2, bias)
    assert idx[0].tolist() == [2, 0]
    e = np.exp(np.array([0.0, 1.0]))
    np.testing.assert_allclose(g[0], e / e.sum(), rtol=1e-15)


def test_topk_alternatives():
    keys = np.array([3.0, 2.0, 1.0, 1.0 + 5e-5, 0.0])
    alts = oracle.topk_alternatives(keys, 3, 1e-4)
    assert sorted(alts) == [(0, 1, 2), (0, 1, 3)]
    assert oracle.topk_alternatives(keys, 2, 1e-4) == [(0, 1)]


# ------------------------------------------------------------------ linear maps (a1, a4, a6, a7, a10)
@pytest.mark.parametrize("fn,out_dim,in_dim", [
    (oracle.router_logits, 6, 10), (oracle.pooler, 5, 10), (oracle.unpooler, 10, 5)])
def test_linear_layers_use_out_by_in_storage(fn, out_dim, in_dim):
    # weights are stored [out, in] (a bias-free linear layer; the deep dive §4.3 gives
    # gate_up_proj as [256, 8192, 4096] = [experts, out, in]); a one-hot weight W[i, j] = 1
    # must carry input coordinate j to output coordinate i.
    W = np.zeros((out_dim, in_dim))
    W[2, 3] = 1.0
    x = np.zeros((1, in_dim))
    x[0, 3] = 5.0
    out = fn(x, W)
    expect = np.zeros((1, out_dim))
    expect[0, 2] = 5.0
    np.testing.assert_array_equal(out, expect)


def test_expert_swiglu_values_and_orientation():
    L = I = 4
    Wg, Wu, Wd = np.zeros((I, L)), np.zeros((I, L)), np.zeros((L, I))
    Wg[1, 0] = 1.0          # gate unit 1 reads z[0]
    Wu[1, 0] = 3.0          # up unit 1 reads 3 z[0]
    Wd[2, 1] = 1.0          # output 2 reads hidden unit 1
    z = np.array([[2.0, 0, 0, 0]])
    y = oracle.expert_ffn(z, Wg, Wu, Wd)
    # E(z) = W_down(SiLU(W_gate z) * W_up z): a = 2, u = 6, h = SiLU(2) * 6 (closed form)
    silu2 = 2.0 / (1.0 + math.exp(-2.0))
    expect = np.zeros((1, L))
    expect[0, 2] = silu2 * 6.0
    np.testing.assert_allclose(y, expect, rtol=1e-15, atol=0)
    # SiLU goes on the gate, not the up projection
    assert abs(y[0, 2] - 2.0 * (6.0 / (1 + math.exp(-6.0)))) > 1.0


def test_silu_closed_forms():
    assert oracle.silu(np.array([0.0]))[0] == 0.0
    assert abs(oracle.silu(np.array([1.0]))[0] - 1.0 / (1.0 + math.exp(-1.0))) < 1e-16
    assert abs(oracle.silu(np.array([-40.0]))[0]) < 1e-15
    assert abs(oracle.silu(np.array([40.0]))[0] - 40.0) < 1e-12


# ------------------------------------------------------------------ whole block
def _random_block(T=7, D=24, L=16, I=12, E=5, seed=0):
    r = np.random.default_rng(seed)
    return dict(x=r.normal(size=(T, D)), W_router=r.normal(size=(E, D)) / math.sqrt(D),
                W_pool=r.normal(size=(L, D)) / math.sqrt(D),
                W_gate=r.normal(size=(E, I, L)) / math.sqrt(L), W_up=r.normal(size=(E, I, L)) / math.sqrt(L),
                W_down=r.normal(size=(E, L, I)) / math.sqrt(I), gamma=r.normal(size=(E, L)) * 0.3,
                W_unpool=r.normal(size=(D, L)) / math.sqrt(L))


def _fwd(b, k, eps=1e-6, **kw):
    return oracle.latent_moe_forward(b["x"], b["W_router"], b["W_pool"], (b["W_gate"], b["W_up"], b["W_down"]),
                                     b["gamma"], b["W_unpool"], k, eps, **kw)


def test_all_experts_identical_k_equals_E_is_one_dense_expert():
    b = _random_block()
    E = b["W_gate"].shape[0]
    for name in ("W_gate", "W_up", "W_down", "gamma"):
        b[name] = np.repeat(b[name][:1], E, axis=0)
    got = _fwd(b, k=E)["out"]
    z = b["x"] @ b["W_pool"].T
    a, u = z @ b["W_gate"][0].T, z @ b["W_up"][0].T
    y = (a / (1 + np.exp(-a)) * u) @ b["W_down"][0].T
    n = y / np.sqrt(np.mean(y * y, 1, keepdims=True) + 1e-6) * (1 + b["gamma"][0])
    np.testing.assert_allclose(got, n @ b["W_unpool"].T, rtol=1e-12, atol=1e-12)


def test_token_permutation_equivariance():
    b = _random_block(T=11)
    ref = _fwd(b, k=2)
    perm = np.random.default_rng(5).permutation(11)
    b2 = dict(b, x=b["x"][perm])
    got = _fwd(b2, k=2)
    np.testing.assert_allclose(got["out"], ref["out"][perm], rtol=1e-13, atol=1e-13)
    np.testing.assert_array_equal(got["idx"], ref["idx"][perm])


def test_down_projection_scale_cancels_in_norm():
    b = _random_block()
    ref = _fwd(b, k=3, eps=0.0)["out"]
    b2 = dict(b, W_down=b["W_down"] * np.array([0.5, 2.0, 3.0, 10.0, 0.1])[:, None, None])
    np.testing.assert_allclose(_fwd(b2, k=3, eps=0.0)["out"], ref, rtol=1e-11, atol=1e-12)


def test_per_expert_gain_is_taken_from_the_selected_expert():
    b = _random_block(T=3, E=4)
    res = _fwd(b, k=2)
    t, j = 1, 1
    e = int(res["idx"][t, j])
    y = res["y"][t, j]
    np.testing.assert_allclose(res["n"][t, j], y / math.sqrt(np.mean(y * y) + 1e-6) * (1 + b["gamma"][e]),
                               rtol=1e-14)
    # shared gain = broadcast of one [L] vector (pages' post_expert_norm)
    shared = oracle.latent_moe_forward(b["x"], b["W_router"], b["W_pool"], (b["W_gate"], b["W_up"], b["W_down"]),
                                       b["gamma"][0], b["W_unpool"], 2, 1e-6)
    np.testing.assert_allclose(shared["n"][t, j], y / math.sqrt(np.mean(y * y) + 1e-6) * (1 + b["gamma"][0]),
                               rtol=1e-14)


def test_callable_expert_source_matches_arrays():
    b = _random_block()
    ref = _fwd(b, k=2)["out"]
    got = oracle.latent_moe_forward(b["x"], b["W_router"], b["W_pool"],
                                    lambda e: (b["W_gate"][e], b["W_up"][e], b["W_down"][e]),
                                    b["gamma"], b["W_unpool"], 2, 1e-6)["out"]
    np.testing.assert_array_equal(got, ref)


# ------------------------------------------------------------------ accounting
def test_parameter_and_flop_accounting():
    a = {s.split()[0]: float(s.split()[1]) for s in lines("accounting.txt")}
    D, L, I, E, k = (int(a[n]) for n in "D L I E k".split())
    assert oracle.expert_param_count(L, I) == a["params_per_expert"]
    assert E * oracle.expert_param_count(L, I) == a["params_all_experts"]
    assert E * D + 2 * D * L + 2 * L == a["params_router_proj_norms"]
    flops = oracle.moe_flops_per_token(D, L, I, E, k)
    # 2 x active parameters, less the two 4096-entry norm gains the FLOP count leaves out
    assert flops == 2 * (a["params_active_per_token"] - 2 * L)
    assert round(flops / 1e6, 1) == a["moe_mflops_per_token_printed"]


# ------------------------------------------------------------------ NVFP4 decoding
def test_e2m1_table():
    for s in lines("fp4_e2m1.txt"):
        code, val = s.split()
        got = oracle.decode_e2m1(int(code))
        assert got == float(val) and np.signbit(got) == val.startswith("-")


def test_e4m3_values_and_every_byte_against_torch():
    for s in lines("fp8_e4m3.txt"):
        b, val = s.split()
        got = float(oracle.decode_e4m3(int(b, 16)))
        assert (np.isnan(got) and val == "nan") or got == float(val)
    import torch
    allb = torch.arange(256, dtype=torch.uint8)
    ref = allb.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle.decode_e4m3(np.arange(256))
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(got[~np.isnan(got)], ref[~np.isnan(ref)])


def test_nibble_order_and_dequantisation():
    codes = np.array([[0x21, 0xF7]], dtype=np.uint8)          # values 1,2 | 7,15
    assert oracle.unpack_nibbles(codes).tolist() == [[1, 2, 7, 15]]
    # one row of 16 weights: codes 0..15, block scale 2.0 (0x40), matrix scale 0.25
    packed = np.array([[lo | (hi << 4) for lo, hi in zip(range(0, 16, 2), range(1, 16, 2))]], dtype=np.uint8)
    w = oracle.dequantize_nvfp4(packed, np.array([[0x40]], dtype=np.uint8), 0.25)
    table = np.array([float(s.split()[1]) for s in lines("fp4_e2m1.txt")])
    np.testing.assert_array_equal(w[0], table * 2.0 * 0.25)


def test_nvfp4_bytes_per_weight():
    # deep dive §7.3: 0.5625 bytes per weight (4 bits + one FP8 scale per 16 weights)
    assert oracle.NVFP4_BYTES_PER_WEIGHT == 0.5625
    out, k = 64, 256
    assert (out * k // 2 + out * k // 16) / (out * k) == 0.5625


# ----------------------------------------------- feed-forward sublayer around the block
def _decimals(s):
    return len(s.split(".")[1]) if "." in s else 0


def test_residual_gate_table():
    """Every row of the gate table (deep dive §5.2): beta, alpha, alpha^2 + beta^2 and the
    rotation angle, each to one unit in its last printed digit."""
    rows = list(lines("residual_gate.txt"))
    assert len(rows) == 5
    for s in rows:
        f = s.split()
        g = float(f[0])
        alpha, beta = oracle.residual_gate_coefficients(np.array([g]))
        got = [beta[0], alpha[0], alpha[0] ** 2 + beta[0] ** 2, math.degrees(math.atan2(beta[0], alpha[0]))]
        for printed, v in zip(f[1:], got):
            assert abs(v - float(printed)) <= 10.0 ** -_decimals(printed), (g, printed, v)


def test_residual_gate_four_channel_example():
    x = np.array([1.0, -1.0, 1.0, -1.0])
    f = np.array([1.0, 1.0, -1.0, -1.0])
    for s in lines("residual_gate_example.txt"):
        v = floats(s)
        out = oracle.residual_gate(x, f, np.full(4, v[0]))
        np.testing.assert_allclose(out, v[1:5], atol=1e-3)
        assert abs(math.sqrt(np.mean(out * out)) - v[5]) <= 1e-3
    # plain addition leaves the unit circle (RMS 1.414 on the page)
    assert abs(math.sqrt(np.mean((x + f) ** 2)) - 1.414) <= 1e-3


def test_residual_gate_floor_and_norm_preservation():
    """alpha^2 + beta^2 = 1 exactly while the floor is inactive, which the page places at
    beta > 0.9995, i.e. g > 2.28; above it alpha stays sqrt(1e-3) and the sum tends to
    1.001. A gate of unit-RMS orthogonal inputs keeps RMS 1 (deep dive §5.2)."""
    g = np.linspace(-6.0, 2.27, 2001)
    a, b = oracle.residual_gate_coefficients(g)
    np.testing.assert_allclose(a * a + b * b, 1.0, rtol=0, atol=1e-13)
    a, b = oracle.residual_gate_coefficients(np.array([2.29, 5.0, 40.0]))
    np.testing.assert_allclose(a, math.sqrt(1e-3), rtol=1e-13)
    assert np.all(a * a + b * b > 1.0) and abs(a[-1] ** 2 + b[-1] ** 2 - 1.001) < 1e-12
    # threshold where sigmoid(-w)(1 + sigmoid(w)) = 1e-3, to the page's two decimals
    thr = 0.3 * math.log(math.sqrt(0.999) / (1.0 - math.sqrt(0.999)))
    assert round(thr, 2) == 2.28
    # a beta of 0.5 sits at g = 0, and beta -> 0 passes the residual stream unchanged
    assert oracle.residual_gate_coefficients(np.array([0.0]))[1][0] == 0.5
    x = RNG.normal(size=64)
    np.testing.assert_allclose(oracle.residual_gate(x, RNG.normal(size=64), np.full(64, -30.0)), x, atol=1e-12)
    # rotation: orthogonal unit-RMS x and f (Hadamard rows) keep RMS 1 for any gate value
    # shared by the channels (the page's example); the cross terms cancel over channels
    h = np.array([[1, 1, 1, 1], [1, -1, 1, -1], [1, 1, -1, -1], [1, -1, -1, 1]], dtype=float)
    for gv in RNG.uniform(-2.0, 2.2, size=20):
        for i, j in ((1, 2), (0, 3), (2, 3)):
            out = oracle.residual_gate(h[i], h[j], np.full(4, gv))
            assert abs(np.mean(out * out) - 1.0) < 1e-13


def test_sublayer_pre_norm_makes_the_block_scale_invariant():
    """With the centred pre-norm (gain 0, eps 0) the block sees x / rms(x), so scaling the
    residual stream leaves the branch output unchanged; without it the output is not."""
    b = _random_block(T=9)
    kw = dict(ffn_pre_gain=np.zeros(b["x"].shape[1]), ffn_pre_eps=0.0)
    ref = _fwd(b, k=2, **kw)
    got = _fwd(dict(b, x=3.7 * b["x"]), k=2, **kw)
    np.testing.assert_allclose(got["f"], ref["f"], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(np.sqrt(np.mean(ref["xn"] ** 2, axis=1)), 1.0, atol=1e-12)
    assert not np.allclose(_fwd(dict(b, x=3.7 * b["x"]), k=2)["out"], _fwd(b, k=2)["out"])


def test_sublayer_post_norm_and_gate():
    """The post-norm branch has RMS sqrt(ms / (ms + eps)) whatever the block computed (the
    page's unit-RMS write, §5.3), its direction is f * (1 + w); a gate of beta -> 0 returns
    the residual stream and of beta -> 1 (floor off) the normalised branch."""
    b = _random_block(T=7)
    D = b["x"].shape[1]
    w = RNG.normal(size=D) * 0.3
    r = _fwd(b, k=2, ffn_post_gain=w, ffn_post_eps=1e-8)
    v = r["f"] * (1 + w)
    ms = np.mean(v * v, axis=1)
    np.testing.assert_allclose(np.sqrt(np.mean(r["out"] ** 2, axis=1)), np.sqrt(ms / (ms + 1e-8)), rtol=1e-12)
    cos = np.sum(r["out"] * v, axis=1) / np.linalg.norm(r["out"], axis=1) / np.linalg.norm(v, axis=1)
    np.testing.assert_allclose(cos, 1.0, atol=1e-12)
    low = _fwd(b, k=2, ffn_post_gain=w, gate=np.full(D, -40.0))
    np.testing.assert_allclose(low["out"], b["x"], atol=1e-12)
    # g = 12: beta = 1 - 4e-18, alpha = 2.9e-9 once the floor is switched off
    high = _fwd(b, k=2, ffn_post_gain=w, gate=np.full(D, 12.0), gate_floor=0.0)
    np.testing.assert_allclose(high["out"], r["out"], atol=1e-7)


def test_round_bf16_against_torch_and_ties():
    """Nearest bfloat16, ties to even: equal to torch's float32 -> bfloat16 conversion on
    float32 inputs, and the hand cases of the 8-bit significand."""
    import torch
    v = RNG.normal(size=20000) * np.exp(RNG.uniform(-20, 20, size=20000))
    v32 = v.astype(np.float32).astype(np.float64)
    ref = torch.from_numpy(v32).to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(oracle.round_bf16(v32), ref)
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: ties to the even significand (1)
    assert oracle.round_bf16(1.0 + 2.0 ** -8) == 1.0
    # 1 + 3 * 2^-8 is halfway between 1 + 2^-7 and 1 + 2^-6: ties to 1 + 2^-6
    assert oracle.round_bf16(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6
    assert oracle.round_bf16(1.0 + 2.0 ** -8 + 2.0 ** -30) == 1.0 + 2.0 ** -7
    assert oracle.round_bf16(-3.0) == -3.0 and oracle.round_bf16(0.0) == 0.0


# ------------------------------------------------------------- NVFP4 activations (W4A4)
def test_e2m1_rounding_table():
    for s in lines("e2m1_rounding.txt"):
        v, code = s.split()
        assert int(oracle.round_e2m1(np.float32(float(v)).astype(np.float64))) == int(code), s


def test_e2m1_rounding_is_nearest_with_ties_to_even():
    """Brute force over random values: the code's value is the nearest E2M1 value, and at
    an exact tie the code with mantissa bit 0 wins."""
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    q = np.concatenate([RNG.uniform(-8, 8, 5000), ties, -ties])
    codes = oracle.round_e2m1(q)
    got = oracle.decode_e2m1(codes)
    allv = oracle.decode_e2m1(np.arange(16))
    for v, c, g in zip(q, codes, got):
        d = np.abs(np.clip(v, -6, 6) - allv)
        assert abs(np.clip(v, -6, 6) - g) <= d.min() + 1e-12
        ties = np.nonzero(np.abs(d - d.min()) < 1e-12)[0]
        if len(set(allv[ties])) > 1:
            assert c & 1 == 0


def test_round_e4m3_against_torch():
    """Nearest E4M3 with ties to even equals torch's float32 -> float8_e4m3fn conversion for
    every value in range, including all exact midpoints between neighbours."""
    import torch
    tab = oracle.decode_e4m3(np.arange(127))
    mids = (tab[:-1] + tab[1:]) / 2
    v = np.concatenate([RNG.uniform(0, 448, 20000), np.exp(RNG.uniform(-12, 6, 20000)), mids, tab]).astype(np.float32)
    v = v[v <= 448]
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(oracle.round_e4m3(v.astype(np.float64)), ref)
    assert int(oracle.round_e4m3(np.array([1000.0]))[0]) == 0x7E          # saturates at 448


def test_activation_quantiser_properties():
    """Per block of 16: the scale is E4M3(amax / 6); the block's largest magnitude maps to
    code 6 or 7 (4 or 6 times the scale); values already on the grid of a block come back
    exactly; a zero block gives zero codes and scale; low nibble = even element."""
    x = RNG.normal(size=(5, 64)).astype(np.float32)
    codes, sc = oracle.quantize_activations_nvfp4(x)
    assert codes.shape == (5, 32) and sc.shape == (5, 4)
    amax = np.abs(x.reshape(5, 4, 16)).max(-1)
    np.testing.assert_array_equal(sc, oracle.round_e4m3((amax / np.float32(6)).astype(np.float32).astype(np.float64)))
    deq = oracle.dequantize_activations_nvfp4(codes, sc).reshape(5, 4, 16)
    top = np.argmax(np.abs(x.reshape(5, 4, 16)), -1)
    ratio = np.abs(np.take_along_axis(deq, top[..., None], -1)[..., 0]) / oracle.decode_e4m3(sc)
    assert np.all((ratio == 4.0) | (ratio == 6.0))
    # a block whose values are E2M1 values times an E4M3 scale of amax/6 round-trips exactly
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6, -.5, -1, -1.5, -2, -3, -4, -6, 6], dtype=np.float32) * np.float32(0.375)
    c2, s2 = oracle.quantize_activations_nvfp4(grid[None, :])
    np.testing.assert_array_equal(oracle.dequantize_activations_nvfp4(c2, s2)[0], grid)
    c3, s3 = oracle.quantize_activations_nvfp4(np.zeros((1, 16), np.float32))
    assert not c3.any() and not s3.any()
    c4, _ = oracle.quantize_activations_nvfp4(np.array([[6, -6] + [0] * 14], np.float32))
    assert c4[0, 0] == 0x7 | (0xF << 4)


def test_w4a4_expert_matches_dequantised_operands():
    """The W4A4 expert equals the plain expert run on quantise-dequantised operands, and
    its error against the unquantised expert is of the size 4-bit activations give."""
    b = _random_block(T=6, D=32, L=32, I=48, E=3)
    ref = _fwd(b, k=2)
    got = _fwd(b, k=2, act_format="nvfp4")
    rel = np.linalg.norm(got["y"] - ref["y"]) / np.linalg.norm(ref["y"])
    assert 0.01 < rel < 0.3
    z = b["x"] @ b["W_pool"].T
    e = int(got["idx"][0, 0])
    zq = oracle.nvfp4_activation(z[:1])
    a = zq @ b["W_gate"][e].T
    h = oracle.nvfp4_activation(a / (1 + np.exp(-a)) * (zq @ b["W_up"][e].T))
    np.testing.assert_allclose(got["y"][0, 0], (h @ b["W_down"][e].T)[0], rtol=1e-12, atol=1e-12)


def test_activation_quantiser_adopts_only_boundary_decisions():
    """Another implementation's decision is adopted only where the input sits within 2^-7 of
    the rounding boundary between two adjacent values; any other difference is an error."""
    base = np.zeros((1, 16), np.float32)
    base[0, 0] = 3.0                            # amax 3 -> scale E4M3(0.5) = 0x30, exact
    own_c, own_s = oracle.quantize_activations_nvfp4(base)
    n = [0]
    c, s = oracle.quantize_activations_nvfp4(base, ref=(own_c, own_s), adopted=n)
    assert n[0] == 0 and np.array_equal(c, own_c) and np.array_equal(s, own_s)

    def with_code(x, i, code):
        c0, s0 = oracle.quantize_activations_nvfp4(x)
        u = oracle.unpack_nibbles(c0)
        u[0, i] = code
        return (u[:, 0::2] | (u[:, 1::2] << 4)).astype(np.uint8), s0

    near = base.copy()
    near[0, 1] = np.float32(0.5 * 1.2501)       # q = 1.2501: just above the 1 / 1.5 midpoint -> 1.5
    assert oracle.unpack_nibbles(oracle.quantize_activations_nvfp4(near)[0])[0, 1] == 3
    n = [0]
    c, _ = oracle.quantize_activations_nvfp4(near, ref=with_code(near, 1, 2), adopted=n)
    assert n[0] == 1 and oracle.unpack_nibbles(c)[0, 1] == 2
    far = base.copy()
    far[0, 1] = np.float32(0.5 * 1.4)           # q = 1.4: well inside the 1.5 interval
    with pytest.raises(ValueError):
        oracle.quantize_activations_nvfp4(far, ref=with_code(far, 1, 2))
    with pytest.raises(ValueError):             # code 5 (value 3) is not a neighbour of 3 (value 1.5)
        oracle.quantize_activations_nvfp4(near, ref=with_code(near, 1, 5))
    # a scale near the midpoint of E4M3 0.5 (0x30) and 0.5625 (0x31): amax / 6 = 0.53126
    sc = np.zeros((1, 16), np.float32)
    sc[0, 0] = np.float32(6 * 0.53126)
    _, s_own = oracle.quantize_activations_nvfp4(sc)
    assert s_own[0, 0] == 0x31
    forced = sc.copy()
    n = [0]
    ref_c = oracle.quantize_activations_nvfp4(forced)[0]
    # the other implementation chose 0x30 and coded the block with it (6.37 -> saturates at 6)
    q_other = np.array([[0x7] + [0] * 7], np.uint8)
    c, s = oracle.quantize_activations_nvfp4(sc, ref=(q_other, np.array([[0x30]], np.uint8)), adopted=n)
    assert s[0, 0] == 0x30 and n[0] == 1
    with pytest.raises(ValueError):             # a scale two steps away is never adopted
        oracle.quantize_activations_nvfp4(sc, ref=(ref_c, np.array([[0x2F]], np.uint8)))
