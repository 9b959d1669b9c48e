"""GPU parity: the CUDA path (through the C ABI) against the FP64 oracle on the same
seeded inputs. Every workload is compared element by element on every token: small ones
on every intermediate, the full-size layers (T=64 decode with BF16 and NVFP4 experts, T=8192
prefill with uniform and Zipf-skewed routing, T=4096 NVFP4 experts as W4A16 and W4A4) on
every routing decision, the permutation, the pooler output, every expert-output row with its
sum of squares, the combined latent and the block output.
"""
import dataclasses

import numpy as np
import pytest
import torch

import latent_mixture_experts_moe_b200 as moe
import oracle
import workloads as W
from parity_util import (Run, assert_close, check_every_token, check_routing, expected_permutation, host,
                         oracle_block, oracle_on_gpu_alternatives)

pytestmark = pytest.mark.gpu


def full_check(w, inp, run, rows=None, **oracle_modes):
    """Routing, permutation, intermediates and output of `run` against the oracle."""
    T = run.T
    rows = np.arange(T) if rows is None else rows
    ref = oracle_block(w, inp, rows, **oracle_modes)
    gidx = run.idx.cpu().numpy()[rows]
    gg = run.g.cpu().numpy()[rows]
    alts = check_routing(ref, gidx, gg, w.k)
    ref_out = oracle_on_gpu_alternatives(w, inp, rows, ref, gidx, alts, **oracle_modes)
    out = host(run.out)[rows]
    assert_close(out, ref_out, f"{w.name} out")
    return ref, alts


# ------------------------------------------------------------------------- small, exact
@pytest.fixture(scope="module")
def tiny():
    w = W.WORKLOADS["tiny"]
    return w, W.make_inputs(w, "cuda")


@pytest.fixture(scope="module")
def mid():
    w = W.WORKLOADS["mid"]
    return w, W.make_inputs(w, "cuda")


@pytest.mark.parametrize("name", ["tiny", "mid"])
def test_small_workload_every_intermediate(name, tiny, mid):
    w, inp = {"tiny": tiny, "mid": mid}[name]
    run = Run(w, inp)
    ref, alts = full_check(w, inp, run)
    act = run.act()
    T, k, L, I, E = w.T, w.k, w.L, w.I, w.E
    # router logits
    logits = run.inter("logits", torch.float32, (T, E)).cpu().numpy()
    assert_close(logits, ref["logits"], "logits", rel=1e-4, max_abs_rms=1e-3)
    # pooler
    assert_close(host(run.inter("z", act, (T, L))), ref["z"], "z")
    if alts:
        return
    counts, offsets, inv = expected_permutation(ref["idx"], E)
    R = run.layout["rows"]
    assert np.array_equal(run.inter("expert_count", torch.int32, (E,)).cpu().numpy(), counts)
    assert np.array_equal(run.inter("expert_offset", torch.int32, (E + 1,)).cpu().numpy(), offsets)
    ginv = run.inter("inv", torch.int32, (T * k,)).cpu().numpy()
    assert np.array_equal(ginv, inv)
    rtok = run.inter("row_token", torch.int32, (R,)).cpu().numpy()
    assert np.array_equal(rtok[inv], np.arange(T * k) // k)
    # expert outputs before the norm, in expert order
    y = host(run.inter("y", act, (R, L)))[ginv].reshape(T, k, L)
    assert_close(y, ref["y"], "y")
    # rows of assignments only (padding rows hold whatever the workspace held)
    ss = run.inter("ss", torch.float32, (R, L // 32)).cpu().numpy()[ginv].astype(np.float64).sum(1).reshape(T, k)
    assert_close(ss, ref["ss"], "sum of squares", rel=2e-2)
    assert_close(host(run.inter("c", act, (T, L))), ref["c"], "combined latent")


def test_repeat_runs_are_bitwise_identical(mid):
    w, inp = mid
    a = Run(w, inp)
    b = Run(w, inp)
    assert torch.equal(a.out, b.out)
    assert torch.equal(a.idx, b.idx) and torch.equal(a.g, b.g)


def test_host_io_entry_point_matches_device_entry_point(mid):
    w, inp = mid
    run = Run(w, inp)
    x_host = inp["x"].cpu().pin_memory()
    out_host = torch.empty((w.T, w.D), dtype=inp["x"].dtype).pin_memory()
    x_dev = torch.empty_like(inp["x"])
    out_dev = torch.empty((w.T, w.D), dtype=inp["x"].dtype, device="cuda")
    cfg = run.model.config(w.T, run.model.workspace)
    moe.forward_host_io(cfg, x_host, x_dev, inp["W_router"], inp["W_pool"], inp["W_gate"], inp["W_up"],
                        inp["W_down"], inp["gamma"], inp["W_unpool"], out_dev, out_host)
    torch.cuda.synchronize()
    assert torch.equal(out_host, run.out.cpu())


# ------------------------------------------------------------- W4A4 (NVFP4 activations)
def test_nvfp4_activation_quantiser_bit_exact():
    """The C-ABI quantiser against the oracle's on the same seeded bf16 rows: every code and
    scale byte equal (rows of N(0, 1) values, of tiny values near the E4M3 subnormals, of
    large values, and all-zero blocks)."""
    w = W.Workload("quant", T=64, D=256, L=256, I=256, E=2, k=1, dtype="bf16", seed=21)
    x = W.make_tensor(w, "x", "cuda")                           # [64, 256] bf16
    x[8:16] *= 1e-3
    x[16:24] *= 60.0
    x[24, :16] = 0.0
    x[25] = 0.0
    codes = torch.empty((64, 128), dtype=torch.uint8, device="cuda")
    scales = torch.empty((64, 16), dtype=torch.uint8, device="cuda")
    moe.quantize_nvfp4_rows(x, codes, scales)
    torch.cuda.synchronize()
    ref_c, ref_s = oracle.quantize_activations_nvfp4(host(x))
    np.testing.assert_array_equal(scales.cpu().numpy(), ref_s)
    np.testing.assert_array_equal(codes.cpu().numpy(), ref_c)


W4A4 = [
    # name, T, D, L, I, E, k
    ("w4a4_tiles128", 256, 1024, 512, 512, 16, 4),
    ("w4a4_tiles32", 16, 1024, 512, 512, 32, 2),
    ("w4a4_ragged", 300, 512, 256, 768, 8, 3),
    # several tiles per CTA and K = 2048: the stage and scale-slot rings wrap many times
    ("w4a4_many_tiles", 2048, 512, 2048, 2048, 64, 4),
]


@pytest.mark.parametrize("case", W4A4, ids=[c[0] for c in W4A4])
def test_w4a4_experts(case):
    """NVFP4 weights and activations (tcgen05 kind::mxf4nvf4) against the oracle running the
    same quantiser on its own activations and the dequantised weight codes."""
    name, T, D, L, I, E, k = case
    w = W.Workload(name, T=T, D=D, L=L, I=I, E=E, k=k, dtype="bf16", seed=13, experts="nvfp4", act="nvfp4")
    inp = W.make_inputs(w, "cuda")
    run = Run(w, inp)
    assert moe.stages(run.model.config(T))[6:9] == ("quant_z", "gather_codes", "gate_up_swiglu")
    rows = np.arange(T)
    ref = oracle_block(w, inp, rows, run=run)
    gidx = run.idx.cpu().numpy()
    alts = check_routing(ref, gidx, run.g.cpu().numpy(), w.k)
    ref_out = oracle_on_gpu_alternatives(w, inp, rows, ref, gidx, alts, run=run)
    r, _ = assert_close(host(run.out), ref_out, f"{name} out", rel=NVFP4_REL_L2)
    decisions = T * k * (L + I) * 17 // 16          # codes and block scales of z and h
    print(f"{name}: rel-L2 {r:.2e}; boundary decisions adopted {ref['act_adopted']} of {decisions}")
    assert ref["act_adopted"] <= 1e-3 * decisions
    if not alts:
        R = run.layout["rows"]
        ginv = run.inter("inv", torch.int32, (T * k,)).cpu().numpy()
        y = host(run.inter("y", torch.bfloat16, (R, L)))[ginv].reshape(T, k, L)
        assert_close(y, ref["y"], f"{name} expert outputs", rel=NVFP4_REL_L2)
        # the quantised latent rows in expert order: every scale byte equal to the oracle's
        # quantisation of its own bf16-rounded z, codes equal except where the two bf16 values
        # of z differ (a float32 vs float64 accumulation crossing a bf16 rounding boundary)
        zq_s = run.inter("zq_scales", torch.uint8, (R, L // 16)).cpu().numpy()[ginv]
        ref_c, ref_s = oracle.quantize_activations_nvfp4(oracle.round_bf16(np.repeat(ref["z"], k, axis=0)))
        assert np.mean(zq_s != ref_s) < 1e-3


@pytest.mark.slow
def test_full_size_w4a4_layer_every_token():
    """The T=4096 layer with NVFP4 weights and activations: every token and every
    assignment row against the oracle on the same codes (2e-2, the NVFP4 tolerance)."""
    w = W.WORKLOADS["nvfp4_w4a4"]
    inp = W.make_inputs(w, "cuda")
    run = Run(w, inp)
    res = check_every_token(w, inp, run, rel=NVFP4_REL_L2)
    decisions = w.T * w.k * (w.L + w.I) * 17 // 16
    print(f"w4a4 full layer: {res}; boundary decisions adopted {res['act_adopted']} of {decisions}")
    assert res["act_adopted"] <= 1e-3 * decisions


def test_host_batches_entry_point_matches_device_forwards(mid):
    """Three different batches through the overlapped host-buffer call give, bit for bit,
    the outputs of three device forwards."""
    w, inp = mid
    import dataclasses
    model = moe.LatentMoE({n: v for n, v in inp.items() if n != "x"}, T_max=w.T, k=w.k, eps=w.eps)
    xs = [W.make_inputs(dataclasses.replace(w, seed=s), "cuda", names=["x"])["x"] for s in (31, 32, 33)]
    want = [model(x.clone()) for x in xs]
    torch.cuda.synchronize()
    x_hosts = [x.cpu().pin_memory() for x in xs]
    out_hosts = [torch.empty((w.T, w.D), dtype=torch.bfloat16).pin_memory() for _ in xs]
    x_devs = [torch.empty_like(xs[0]) for _ in range(2)]
    out_devs = [torch.empty((w.T, w.D), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    cfg = model.config(w.T, model.workspace)
    wt = model.w
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    moe.forward_host_batches(cfg, x_hosts, out_hosts, x_devs, out_devs, wt["W_router"], wt["W_pool"], wt["W_gate"],
                             wt["W_up"], wt["W_down"], wt["gamma"], wt["W_unpool"], torch.cuda.current_stream(), up,
                             down)
    torch.cuda.synchronize()
    for got, ref in zip(out_hosts, want):
        assert torch.equal(got, ref.cpu())
    code, detail = moe.last_device_status(cfg)
    assert code == 0


# ------------------------------------------------------------------------- CUDA graphs
GRAPH = [
    # name, T, D, L, I, E, k: decode-sized tiles (one-CTA kernels), and CTA-pair tiles whose
    # tile counters must be re-zeroed inside every replay
    ("graph_small_tiles", 96, 1024, 512, 512, 32, 4),
    ("graph_pair_tiles", 1024, 1024, 512, 512, 4, 2),
    # NVFP4 weights and activations (W4A4): its GEMMs claim tiles from counters too
    ("graph_w4a4", 512, 1024, 512, 512, 8, 2),
]


@pytest.mark.parametrize("case", GRAPH, ids=[c[0] for c in GRAPH])
def test_cuda_graph_replay_matches_eager(case):
    """The forward captured once in a CUDA graph and replayed gives the eager result bit for
    bit, also after new tokens are written into the captured input buffer."""
    import dataclasses
    name, T, D, L, I, E, k = case
    w4a4 = name.endswith("w4a4")
    w = W.Workload(name, T=T, D=D, L=L, I=I, E=E, k=k, dtype="bf16", seed=11,
                   experts="nvfp4" if w4a4 else "bf16", act="nvfp4" if w4a4 else "bf16")
    inp = W.make_inputs(w, "cuda")
    modes = {"act_format": moe.ACT_NVFP4} if w4a4 else {}
    model = moe.LatentMoE({n: v for n, v in inp.items() if n != "x"}, T_max=T, k=k, eps=w.eps, **modes)
    x = inp["x"].clone()
    out_g = torch.empty((T, D), dtype=torch.bfloat16, device="cuda")
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        model(x, out=out_g)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        model(x, out=out_g)
    x2 = W.make_inputs(dataclasses.replace(w, seed=12), "cuda", names=["x"])["x"]
    for xs in (inp["x"], x2, inp["x"]):
        x.copy_(xs)
        graph.replay()
        torch.cuda.synchronize()
        eager = model(xs.clone())
        torch.cuda.synchronize()
        assert torch.equal(out_g, eager)
    code, detail = moe.last_device_status(model.config(T, model.workspace))
    assert code == 0, f"status {code} detail {detail:#x}"
    del graph


# ------------------------------------------------- feed-forward sublayer around the block
SUBLAYER = [
    # name, T, D, L, I, E, k, dtype, steps (pre-norm, post-norm, residual gate)
    ("sublayer_all_mid", 256, 2048, 1024, 1024, 64, 4, "bf16", ("pre", "post", "gate")),
    ("sublayer_pre_only", 64, 1024, 512, 512, 16, 2, "bf16", ("pre",)),
    ("sublayer_post_gate", 64, 1024, 512, 512, 16, 2, "bf16", ("post", "gate")),
    ("sublayer_gate_only", 48, 1024, 512, 512, 16, 2, "bf16", ("gate",)),
    ("sublayer_all_f32", 37, 256, 256, 128, 8, 3, "f32", ("pre", "post", "gate")),
    # the unpooler on CTA pairs (>= one wave of 256 x 256 tiles) with the squares epilogue
    ("sublayer_all_pair_unpooler", 1280, 4096, 512, 512, 8, 2, "bf16", ("pre", "post", "gate")),
]
SUBLAYER_KEYS = {"pre": "ffn_pre_gain", "post": "ffn_post_gain", "gate": "residual_gate"}


@pytest.mark.parametrize("case", SUBLAYER, ids=[c[0] for c in SUBLAYER])
def test_feedforward_sublayer(case):
    name, T, D, L, I, E, k, dt, steps = case
    w = W.Workload(name, T=T, D=D, L=L, I=I, E=E, k=k, dtype=dt, seed=5)
    inp = W.make_inputs(w, "cuda")
    sub = W.sublayer_inputs(w, "cuda")
    for st in steps:
        inp[SUBLAYER_KEYS[st]] = sub[SUBLAYER_KEYS[st]]
    run = Run(w, inp)
    ref, alts = full_check(w, inp, run)
    cfg = run.model.config(T, run.model.workspace)
    n_launch = moe.launch_count(cfg)
    assert n_launch == 11 + ("pre" in steps) + ("post" in steps or "gate" in steps)
    names = moe.stages(cfg)
    assert len(names) == n_launch
    if "pre" in steps:
        assert names[0] == "ffn_pre_norm"
        xn = host(run.inter("xn", run.act(), (T, D)))
        assert_close(xn, ref["xn"], "xn", rel=5e-3, max_abs_rms=2e-2)
    # every stage event is recorded once per launch, in order
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(n_launch + 1)]
    for e in ev:
        e.record()
    out2 = run.model(inp["x"], stage_events=moe.event_handles(ev))
    torch.cuda.synchronize()
    assert torch.equal(out2, run.out)
    assert all(ev[i].elapsed_time(ev[i + 1]) >= 0.0 for i in range(n_launch))


# ------------------------------------------------------------------------- edge cases
EDGE = [
    # name, T, D, L, I, E, k, dtype, bias_kind
    ("one_token", 1, 256, 128, 128, 8, 2, "bf16", None),
    ("ragged_17", 17, 384, 256, 128, 16, 3, "bf16", None),
    ("ragged_300_wide_I", 300, 256, 128, 384, 8, 2, "bf16", None),
    ("empty_experts", 3, 256, 128, 128, 64, 2, "bf16", None),
    ("expert_takes_all", 300, 256, 128, 128, 8, 2, "bf16", "all_to_0"),
    ("k_equals_E", 40, 256, 128, 256, 4, 4, "bf16", None),
    ("k_one", 33, 256, 256, 128, 16, 1, "bf16", None),
    ("fp32_ragged", 37, 256, 256, 128, 8, 3, "f32", None),
    ("many_tokens_per_expert", 1100, 256, 128, 128, 4, 2, "bf16", None),
    # 256-feature tiles: the unpooler has >= one wave of 256-wide tiles, down has L % 256 == 0;
    # with I % 256 == 0 and L % 512 == 0 gate/up and down run on CTA pairs (cta_group::2)
    ("wide_tiles", 4864, 2048, 512, 256, 8, 2, "bf16", None),
    # CTA pairs with ragged token chunks (about 388 rows per expert in two chunks), down
    # on 256-feature pair tiles (L % 512 != 0)
    ("pair_ragged", 777, 512, 256, 512, 4, 2, "bf16", None),
]


@pytest.mark.parametrize("case", EDGE, ids=[c[0] for c in EDGE])
def test_edge_cases(case):
    name, T, D, L, I, E, k, dt, bias_kind = case
    w = W.Workload(name, T=T, D=D, L=L, I=I, E=E, k=k, dtype=dt, seed=3)
    inp = W.make_inputs(w, "cuda")
    if bias_kind == "all_to_0":
        b = torch.zeros(E, dtype=torch.float32)
        b[0] = 100.0
        inp["router_bias"] = b.cuda()
    run = Run(w, inp)
    ref, alts = full_check(w, inp, run)
    if bias_kind == "all_to_0":
        assert np.all(run.idx.cpu().numpy()[:, 0] == 0)
    if not alts:
        counts, offsets, inv = expected_permutation(ref["idx"], E)
        assert np.array_equal(run.inter("inv", torch.int32, (T * k,)).cpu().numpy(), inv)


# ------------------------------------------------------------------------- failure detection
def test_bounded_wait_times_out_and_the_context_stays_usable(tiny):
    """A wait that nothing completes gives up after its limit and reports
    MUSE_ERR_TIMEOUT through the status word; no trap, no hang, and the next forward runs."""
    status = torch.zeros(2, dtype=torch.int32, device="cuda")
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    moe.selftest_bounded_wait(2_000_000, status)          # 2 ms limit
    end.record()
    torch.cuda.synchronize()
    assert status.tolist() == [5, 0x5E1F]                  # MUSE_ERR_TIMEOUT, the wait's id
    assert start.elapsed_time(end) >= 2.0
    w, inp = tiny
    run = Run(w, inp)                                      # the context is still usable
    full_check(w, inp, run)


def test_selftest_rejects_bad_arguments():
    lib = moe.lib()
    assert lib.muse_selftest_bounded_wait(1000, None, None) == 1
    status = torch.zeros(2, dtype=torch.int32, device="cuda")
    assert lib.muse_selftest_bounded_wait(0, status.data_ptr(), None) == 1
    assert lib.muse_selftest_bounded_wait(10**11, status.data_ptr(), None) == 1


# ------------------------------------------------------------------------- released mode
PAGES = [
    # name, T, D, L, I, E, k
    ("pages_mid", 256, 2048, 1024, 1024, 64, 4),
    ("pages_ragged", 37, 512, 256, 384, 16, 8),
]


@pytest.mark.parametrize("case", PAGES, ids=[c[0] for c in PAGES])
def test_pages_released_mode(case):
    """The block as the pages describe the released model (deep dive §4.2-4.4, Norm
    gates page): sigmoid router on the logits times 1/sqrt(D/256) with a selection-only
    bias and s/(sum s + 1e-15) weights; centred pre-expert norm (eps 1e-5) on z; ONE
    input-scaled post-expert norm gain shared by every expert (eps 1e-8)."""
    name, T, D, L, I, E, k = case
    w = W.Workload(name, T=T, D=D, L=L, I=I, E=E, k=k, dtype="bf16", eps=1e-8, seed=5)
    inp = W.make_inputs(w, "cuda")
    inp["gamma"] = inp["gamma"][0].contiguous()                      # one shared [L] gain
    pre = torch.empty(L, dtype=torch.bfloat16, device="cuda")
    inp["pre_norm_gain"] = W.fill(pre, w.seed, 11, 0.3)
    inp["router_bias"] = (W.normal_f64(w.seed, 12, 0, E) * 0.05).to(torch.float32).cuda()
    scale = 1.0 / np.sqrt(D / 256)
    run = Run(w, inp, router_mode=moe.ROUTER_SIGMOID, router_logit_scale=scale, routed_scaling=1.0,
              norm_mode=moe.NORM_INPUT_SCALED, gamma_shared=True, pre_norm_eps=1e-5)
    ref, alts = full_check(w, inp, run, router_mode="sigmoid", logit_scale=scale, routed_scaling=1.0,
                           norm_mode="input_scaled", pre_norm_eps=1e-5)
    assert_close(host(run.inter("z", run.act(), (T, L))), ref["z"], "normalised latent z")
    g = run.g.cpu().numpy()
    assert np.allclose(g.sum(1), 1.0, atol=1e-5)                     # convex combination


# ------------------------------------------------------------------------- NVFP4 experts
NVFP4 = [
    # name, T, D, L, I, E, k  (bn 32 tiles; bn 256 tiles with 256-feature down tiles; ragged)
    ("nvfp4_mid", 256, 2048, 1024, 1024, 64, 4),
    ("nvfp4_wide", 1100, 512, 512, 512, 4, 2),
    ("nvfp4_ragged", 37, 256, 256, 384, 8, 3),
]
NVFP4_REL_L2 = 2e-2   # the block's NVFP4 tolerance against the oracle on the same codes


@pytest.mark.parametrize("case", NVFP4, ids=[c[0] for c in NVFP4])
def test_nvfp4_experts(case):
    name, T, D, L, I, E, k = case
    w = W.Workload(name, T=T, D=D, L=L, I=I, E=E, k=k, dtype="bf16", seed=9, experts="nvfp4")
    inp = W.make_inputs(w, "cuda")
    run = Run(w, inp)
    rows = np.arange(T)
    ref = oracle_block(w, inp, rows)
    gidx = run.idx.cpu().numpy()
    alts = check_routing(ref, gidx, run.g.cpu().numpy(), w.k)
    ref_out = oracle_on_gpu_alternatives(w, inp, rows, ref, gidx, alts)
    r, _ = assert_close(host(run.out), ref_out, f"{name} out", rel=NVFP4_REL_L2)
    print(f"{name}: rel-L2 {r:.2e}")
    if not alts:
        R = run.layout["rows"]
        ginv = run.inter("inv", torch.int32, (T * k,)).cpu().numpy()
        y = host(run.inter("y", torch.bfloat16, (R, L)))[ginv].reshape(T, k, L)
        assert_close(y, ref["y"], f"{name} expert outputs", rel=NVFP4_REL_L2)


NVFP4_GEMV = [
    # name, T, D, L, I, E, k: a few rows per expert (T*k <= 4E), where both expert GEMMs run
    # on the register-fed MMA kernel -- four rows per expert on average; up to ~10 rows per
    # expert (one or two 8-token groups, ragged) with one 256-element stage past the first
    # in the down projection; a latent of 4608 (18 stages in gate/up)
    ("nvfp4_gemv", 64, 1024, 1024, 1024, 64, 4),
    ("nvfp4_gemv_ragged", 32, 256, 512, 768, 8, 1),
    ("nvfp4_gemv_wide", 6, 256, 4608, 256, 4, 2),
]


@pytest.mark.parametrize("released", [False, True], ids=["centred", "released"])
@pytest.mark.parametrize("case", NVFP4_GEMV, ids=[c[0] for c in NVFP4_GEMV])
def test_nvfp4_decode_sized_experts_every_row(case, released):
    """NVFP4 experts with bf16 activations at decode-sized tiles: out, z, c, every
    assignment row of y and of its sum of squares, and the permutation against the oracle
    (2e-2). The released variant adds the sigmoid router, the pre-expert norm and one
    shared input-scaled post-expert gain (the sums of squares then carry the gain)."""
    name, T, D, L, I, E, k = case
    w = W.Workload(name, T=T, D=D, L=L, I=I, E=E, k=k, dtype="bf16", seed=17, experts="nvfp4")
    if released:
        w = dataclasses.replace(w, eps=1e-8)
    inp = W.make_inputs(w, "cuda")
    if released:
        inp["gamma"] = inp["gamma"][0].contiguous()
        pre = torch.empty(L, dtype=torch.bfloat16, device="cuda")
        inp["pre_norm_gain"] = W.fill(pre, w.seed, 11, 0.3)
        inp["router_bias"] = (W.normal_f64(w.seed, 12, 0, E) * 0.05).to(torch.float32).cuda()
        scale = 1.0 / np.sqrt(D / 256)
        run = Run(w, inp, router_mode=moe.ROUTER_SIGMOID, router_logit_scale=scale, routed_scaling=1.0,
                  norm_mode=moe.NORM_INPUT_SCALED, gamma_shared=True, pre_norm_eps=1e-5)
        res = check_every_token(w, inp, run, rel=NVFP4_REL_L2, router_mode="sigmoid", logit_scale=scale,
                                routed_scaling=1.0, norm_mode="input_scaled", pre_norm_eps=1e-5)
    else:
        run = Run(w, inp)
        res = check_every_token(w, inp, run, rel=NVFP4_REL_L2)
    print(f"{name} ({'released' if released else 'centred'}): {res}")


@pytest.mark.slow
def test_full_size_nvfp4_layer_every_token():
    """The T=4096 layer with NVFP4 expert weights and bf16 activations (W4A16): every token
    and every assignment row against the oracle on the dequantised codes."""
    w = W.WORKLOADS["nvfp4"]
    inp = W.make_inputs(w, "cuda")
    run = Run(w, inp)
    res = check_every_token(w, inp, run, rel=NVFP4_REL_L2)
    print(f"nvfp4 full layer: {res}")


def test_nvfp4_decode_sized_skewed_expert():
    """One expert taking every token (a strong selection bias, sigmoid router): two full
    16-row tiles (two 8-token groups per MMA step), beside experts with a row or two."""
    T, D, L, I, E, k = 32, 256, 512, 512, 16, 2
    w = W.Workload("nvfp4_gemv_skew", T=T, D=D, L=L, I=I, E=E, k=k, dtype="bf16", seed=23, experts="nvfp4")
    inp = W.make_inputs(w, "cuda")
    bias = W.normal_f64(w.seed, 12, 0, E) * 0.05
    bias[3] += 8.0
    inp["router_bias"] = bias.to(torch.float32).cuda()
    run = Run(w, inp, router_mode=moe.ROUTER_SIGMOID, routed_scaling=1.0)
    counts = run.inter("expert_count", torch.int32, (E,)).cpu().numpy()
    assert counts[3] == T and counts.max() == T, counts
    res = check_every_token(w, inp, run, rel=NVFP4_REL_L2, router_mode="sigmoid", routed_scaling=1.0)
    print(f"nvfp4_gemv_skew: {res}")


@pytest.mark.slow
def test_full_size_nvfp4_decode_every_token():
    """The T=64 decode layer with NVFP4 expert weights and bf16 activations (both expert
    GEMMs on the CUDA-core NVFP4 kernel): every token and every assignment row against the
    oracle on the dequantised codes."""
    w = W.WORKLOADS["nvfp4_decode"]
    inp = W.make_inputs(w, "cuda")
    run = Run(w, inp)
    res = check_every_token(w, inp, run, rel=NVFP4_REL_L2)
    print(f"nvfp4 decode layer: {res}")


# ------------------------------------------------------------------------- full size
@pytest.fixture(scope="module")
def full_weights():
    w = W.WORKLOADS["prefill"]
    inp = W.make_inputs(w, "cuda", names=["W_router", "W_pool", "W_gate", "W_up", "W_down", "gamma", "W_unpool"])
    inp["x"] = W.make_tensor(w, "x", "cuda")
    yield inp
    del inp
    torch.cuda.empty_cache()


@pytest.mark.slow
def test_full_size_decode_all_tokens(full_weights):
    w = W.WORKLOADS["decode"]
    run = Run(w, full_weights, T=w.T)
    res = check_every_token(w, full_weights, run)
    print(f"decode: {res}")
    # about 222 distinct experts are touched by 64 tokens x top-8 of 256
    assert 180 <= len(np.unique(run.idx.cpu().numpy())) <= 256


@pytest.mark.slow
@pytest.mark.parametrize("name", ["prefill", "prefill_zipf"])
def test_full_size_prefill_every_token(name, full_weights):
    """The T=8192 layer (uniform routing, and Zipf-skewed through the stored selection
    bias): every token, every assignment row and the permutation against the oracle."""
    w = W.WORKLOADS[name]
    inp = dict(full_weights)
    if w.routing == "zipf":
        inp["router_bias"] = W.zipf_router_bias(w).cuda()
    run = Run(w, inp)
    gpu_logits = run.inter("logits", torch.float32, (w.T, w.E)).cpu().numpy()
    # bf16 products are exact in FP32; FP32 accumulation over D=8192 terms stays far below 1e-3
    ref_logits = oracle.router_logits(host(inp["x"]), host(inp["W_router"]))
    assert np.abs(gpu_logits - ref_logits).max() < 1e-3
    del gpu_logits, ref_logits
    res = check_every_token(w, inp, run)
    # every differing token was checked to be a near tie (gap < 1e-4) with a valid
    # alternative set; the Zipf bias packs keys at the boundary, so they are not rare
    assert res["near_ties"] <= 0.01 * w.T
    print(f"{w.name}: {res}")
    if w.routing == "zipf":
        loads = np.sort(np.bincount(run.idx.cpu().numpy().ravel(), minlength=w.E))[::-1]
        target = W.zipf_target_loads(w.T, w.E, w.k).numpy()
        assert loads[0] >= 0.99 * w.T and loads[1] >= 0.99 * w.T   # water-filled ranks 1-2 take ~every token
        assert np.abs(loads - target).sum() / (w.T * w.k) < 0.02


# ------------------------------------------------------------------- shape-checked boundary
def test_checked_entry_point_rejects_bad_tensors_and_matches_the_raw_one(mid):
    """muse_latent_moe_forward_checked on real device tensors: a weight of the wrong shape, a
    non-contiguous view and an output overlapping the input are each MUSE_ERR_INVALID_ARG with
    nothing launched (the output keeps its contents); correct tensors give the raw entry
    point's output bit for bit."""
    w, inp = mid
    model = moe.LatentMoE({k: v for k, v in inp.items() if k != "x"}, T_max=w.T, k=w.k, eps=w.eps)
    cfg = model.config(w.T, model.workspace)
    ws = [inp[n] for n in ("W_router", "W_pool", "W_gate", "W_up", "W_down", "gamma", "W_unpool")]
    ref = torch.empty((w.T, w.D), dtype=torch.bfloat16, device="cuda")
    moe.forward(cfg, inp["x"], *ws, ref)
    out = torch.empty_like(ref)
    moe.forward_checked(cfg, inp["x"], *ws, out)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    sentinel = torch.full_like(ref, 7.0)
    bad_down = inp["W_down"][:, :, : w.I // 2]                      # [E, L, I/2] view: wrong shape
    bad_pool = inp["W_pool"].t()                                     # transposed view: strides
    cases = {
        "W_down shape": (inp["x"], *ws[:4], bad_down.contiguous(), *ws[5:]),
        "W_pool strides": (inp["x"], ws[0], bad_pool, *ws[2:]),
        "x rows": (inp["x"][: w.T // 2], *ws),
    }
    for name, args in cases.items():
        o = sentinel.clone()
        with pytest.raises(moe.MuseError) as e:
            moe.forward_checked(cfg, *args, o)
        assert e.value.code == 1, name
        torch.cuda.synchronize()
        assert torch.equal(o, sentinel), f"{name}: something was written"
    # out overlapping x
    x2 = inp["x"].clone()
    with pytest.raises(moe.MuseError) as e:
        moe.forward_checked(cfg, x2, *ws, x2)
    assert e.value.code == 1
