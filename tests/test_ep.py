"""Expert parallelism: the exchange orchestration of latent_mixture_experts_moe_b200.ep on
CPU ranks (gloo, uneven token counts, a rank with no tokens), and the library's three EP
entry points on one GPU with the ranks' exchanges done by slicing (no kernel waits on
another). Both compare with the FP64 oracle's single-device forward of the same tokens.

The CPU ranks' compute is a test stand-in written here from the EP contract of
include/muse_moe.h (send rows in expert, token, slot order; expert outputs and per-32-column
partial sums of squares back in the order received; norm and combine on the token's rank),
built from the oracle's steps; it checks that ep_forward routes every row to the rank that
owns its expert and every result back to the row it came from.
"""
import math
import os
import socket

import numpy as np
import pytest
import torch

import oracle
import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleShard:
    """Rank `rank` of G in float64 on the CPU, following the EP contract step by step."""

    def __init__(self, inp, rank, G, k, eps):
        f = oracle.as_f64
        self.Wr, self.Wp, self.Wu = f(inp["W_router"]), f(inp["W_pool"]), f(inp["W_unpool"])
        self.gamma = f(inp["gamma"])
        self.E = self.Wr.shape[0]
        self.E_loc = self.E // G
        lo = rank * self.E_loc
        # this rank holds only its own experts
        self.Wg = f(inp["W_gate"][lo:lo + self.E_loc])
        self.Wup = f(inp["W_up"][lo:lo + self.E_loc])
        self.Wd = f(inp["W_down"][lo:lo + self.E_loc])
        self.G, self.k, self.eps = G, k, eps
        self.L = self.Wp.shape[0]

    def dispatch(self, x):
        x = x.numpy()
        T, k = x.shape[0], self.k
        if T == 0:
            self.pos, self.idx, self.g = {}, np.zeros((0, k), np.int64), np.zeros((0, k))
            return (torch.zeros((0, self.L), dtype=torch.float64), torch.zeros(0, dtype=torch.int32), [0] * self.G)
        self.idx, self.g, _ = oracle.route(oracle.router_logits(x, self.Wr), k)
        z = oracle.pooler(x, self.Wp)
        pairs = sorted((int(self.idx[t, j]), t, j) for t in range(T) for j in range(k))
        self.pos = {(t, j): p for p, (_, t, j) in enumerate(pairs)}
        send_z = np.stack([z[t] for _, t, _ in pairs])
        send_e = np.array([e % self.E_loc for e, _, _ in pairs], dtype=np.int32)
        counts = [sum(1 for e, _, _ in pairs if e // self.E_loc == r) for r in range(self.G)]
        return torch.from_numpy(send_z), torch.from_numpy(send_e), counts

    def experts(self, recv_z, recv_e):
        z, e = recv_z.numpy(), recv_e.numpy()
        y = np.zeros((z.shape[0], self.L))
        for i in range(z.shape[0]):
            y[i] = oracle.expert_ffn(z[i:i + 1], self.Wg[e[i]], self.Wup[e[i]], self.Wd[e[i]])[0]
        ss = (y * y).reshape(y.shape[0], self.L // 32, 32).sum(axis=2)
        return torch.from_numpy(y), torch.from_numpy(ss)

    def combine(self, x, back_y, back_ss):
        T, k = x.shape[0], self.k
        y, ss = back_y.numpy(), back_ss.numpy()
        n = np.zeros((T, k, self.L))
        for t in range(T):
            for j in range(k):
                p = self.pos[(t, j)]
                n[t, j] = oracle.centred_rmsnorm(y[p], self.gamma[self.idx[t, j]], self.eps)
                assert abs(ss[p].sum() - (y[p] ** 2).sum()) <= 1e-9 * max(1.0, ss[p].sum())
        return torch.from_numpy(oracle.unpooler(oracle.combine(n, self.g), self.Wu))


def _tokens(w, counts):
    whole = torch.empty((sum(counts), w.D), dtype=torch.float32)
    W.fill(whole, w.seed, W.TID["x"], 1.0)
    starts = np.concatenate([[0], np.cumsum(counts)])
    return whole, [whole[starts[r]:starts[r + 1]] for r in range(len(counts))]


def _worker(rank, world, port, counts, q):
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from latent_mixture_experts_moe_b200 import ep
        w = W.WORKLOADS["tiny"]
        inp = W.make_inputs(w, "cpu", names=["W_router", "W_pool", "W_gate", "W_up", "W_down", "gamma", "W_unpool"])
        _, xs = _tokens(w, counts)
        shard = OracleShard(inp, rank, world, w.k, w.eps)
        out = ep.ep_forward(shard, xs[rank].to(torch.float64))
        f = oracle.as_f64
        err, n_remote = 0.0, 0
        if counts[rank]:
            ref = oracle.latent_moe_forward(f(xs[rank]), f(inp["W_router"]), f(inp["W_pool"]),
                                            (f(inp["W_gate"]), f(inp["W_up"]), f(inp["W_down"])), f(inp["gamma"]),
                                            f(inp["W_unpool"]), w.k, w.eps)
            err = float(np.abs(out.numpy() - ref["out"]).max())
            n_remote = int(np.sum(ref["idx"] // shard.E_loc != rank))
        q.put((rank, tuple(out.shape), err, n_remote))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("counts", [(5, 11), (3, 0, 7, 5)], ids=["2ranks", "4ranks_one_empty"])
def test_ep_forward_over_gloo_ranks_matches_the_single_device_block(counts):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    world = len(counts)
    procs = [ctx.Process(target=_worker, args=(r, world, port, counts, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=300) for _ in range(world))
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    w = W.WORKLOADS["tiny"]
    for r, shape, err, _ in res:
        assert shape == (counts[r], w.D)
        assert err < 1e-12, f"rank {r}: max error {err}"
    assert sum(n for *_, n in res) > 0  # rows did cross between ranks


# ---------------------------------------------------------------------------------- GPU
EXPERT_KEYS = ("W_gate", "W_up", "W_down")  # dense tensors or their NVFP4 _codes / _scales / _mscale

EP_CASES = [
    # name, workload, ranks, tokens per rank, extra steps ("sublayer": the feed-forward
    # sublayer around the block; "pages": the released model's router and norms)
    ("mid_1rank", W.WORKLOADS["mid"], 1, (96,), None),
    ("mid_2ranks", W.WORKLOADS["mid"], 2, (100, 156), None),
    ("mid_4ranks_one_empty", W.WORKLOADS["mid"], 4, (64, 0, 97, 95), None),
    ("sublayer_2ranks", W.Workload("ep_sublayer", T=256, D=2048, L=1024, I=1024, E=64, k=4, dtype="bf16", seed=5),
     2, (120, 136), "sublayer"),
    ("pages_mode_2ranks", W.Workload("ep_pages", T=256, D=2048, L=1024, I=1024, E=64, k=4, dtype="bf16", eps=1e-8,
                                     seed=5), 2, (140, 116), "pages"),
    ("f32_2ranks", W.Workload("ep_f32", T=37, D=256, L=256, I=128, E=8, k=3, dtype="f32", seed=7), 2, (17, 20),
     None),
    ("nvfp4_w4a16_2ranks", W.Workload("ep_nvfp4", T=200, D=1024, L=512, I=512, E=16, k=4, dtype="bf16", seed=13,
                                      experts="nvfp4"), 2, (90, 110), None),
    ("nvfp4_w4a4_4ranks", W.Workload("ep_w4a4", T=256, D=1024, L=512, I=512, E=16, k=4, dtype="bf16", seed=13,
                                     experts="nvfp4", act="nvfp4"), 4, (70, 58, 64, 64), None),
]


def _shard_weights(inp, r, E_loc):
    """Rank r's weights: everything replicated except its slice of the expert tensors."""
    wts = {}
    for n, v in inp.items():
        if n == "x":
            continue
        if n.startswith(EXPERT_KEYS):
            wts[n] = v[r * E_loc:(r + 1) * E_loc].contiguous()
        else:
            wts[n] = v
    return wts


@pytest.mark.gpu
@pytest.mark.parametrize("case", EP_CASES, ids=[c[0] for c in EP_CASES])
def test_ep_entry_points_on_one_gpu_match_the_oracle_and_the_fused_forward(case):
    import latent_mixture_experts_moe_b200 as moe
    from latent_mixture_experts_moe_b200 import ep
    import parity_util as P
    name, w, G, counts, extra = case
    dev = torch.device("cuda")
    inp = W.make_inputs(w, dev)
    modes, oracle_modes = {}, {}
    if extra == "sublayer":
        inp.update(W.sublayer_inputs(w, dev))
    elif extra == "pages":
        # sigmoid router on logits x 1/sqrt(D/256) with a selection-only bias, centred
        # pre-expert norm, one input-scaled post-expert gain shared by every expert
        inp["gamma"] = inp["gamma"][0].contiguous()
        pre = torch.empty(w.L, dtype=torch.bfloat16, device=dev)
        inp["pre_norm_gain"] = W.fill(pre, w.seed, 11, 0.3)
        inp["router_bias"] = (W.normal_f64(w.seed, 12, 0, w.E) * 0.05).to(torch.float32).to(dev)
        scale = 1.0 / math.sqrt(w.D / 256)
        modes = dict(router_mode=moe.ROUTER_SIGMOID, router_logit_scale=scale, routed_scaling=1.0,
                     norm_mode=moe.NORM_INPUT_SCALED, gamma_shared=True, pre_norm_eps=1e-5)
        oracle_modes = dict(router_mode="sigmoid", logit_scale=scale, routed_scaling=1.0, norm_mode="input_scaled",
                            pre_norm_eps=1e-5)
    T = sum(counts)
    x = inp["x"][:T]
    starts = np.concatenate([[0], np.cumsum(counts)])
    xs = [x[starts[r]:starts[r + 1]] for r in range(G)]
    E_loc = w.E // G
    if w.act == "nvfp4":
        modes = dict(modes, act_format=moe.ACT_NVFP4)
    shards = [ep.ExpertShard(_shard_weights(inp, r, E_loc), r, G, T_max=max(counts), k=w.k, eps=w.eps, **modes)
              for r in range(G)]
    outs = ep.ep_forward_one_device(shards, xs)
    torch.cuda.synchronize()
    for s in shards:
        for ws in (s.ws_home, s.ws_experts):
            code, detail = moe.last_device_status(s.config(1, ws))
            assert code == 0, f"status {code} {detail:#x}"
    got = torch.cat(outs)
    assert got.shape == (T, w.D)
    # the fused single-GPU forward of the same tokens: the same kernels over other row counts,
    # each output element accumulated over K in the same order -- equal bit for bit
    fused = P.Run(w, inp, T=T, **{k: v for k, v in modes.items() if k != "act_format"})
    d = (got.float() - fused.out.float()).abs()
    assert torch.equal(got, fused.out), f"max |EP - fused| = {float(d.max()):.3e}"
    # the oracle, with the routing rule of the parity tests (W4A4: the fused run's activation
    # codes are the candidate decisions at rounding boundaries)
    rows = np.arange(T)
    ref = P.oracle_block(w, inp, rows, run=fused, **oracle_modes)
    alt = P.check_routing(ref, fused.idx.cpu().numpy(), fused.g.cpu().numpy(), w.k)
    want = P.oracle_on_gpu_alternatives(w, inp, rows, ref, fused.idx.cpu().numpy(), alt, run=fused, **oracle_modes)
    P.assert_close(got.double().cpu().numpy(), want, f"EP {name}", rel=2e-2 if w.experts == "nvfp4" else P.REL_L2)
    print(f"{name}: max |EP - fused| = {float(d.max()):.3e}, equal elements {float((d == 0).float().mean()):.4f}")


@pytest.mark.gpu
def test_ep_experts_records_an_out_of_range_local_expert_and_zeroes_its_row():
    import latent_mixture_experts_moe_b200 as moe
    from latent_mixture_experts_moe_b200 import ep
    w = W.WORKLOADS["mid"]
    dev = torch.device("cuda")
    inp = W.make_inputs(w, dev)
    G = 2
    E_loc = w.E // G
    wts = {n: v for n, v in inp.items() if n not in ("x", "W_gate", "W_up", "W_down")}
    for n in ("W_gate", "W_up", "W_down"):
        wts[n] = inp[n][:E_loc].contiguous()
    s = ep.ExpertShard(wts, 0, G, T_max=16, k=w.k, eps=w.eps)
    recv_z = torch.randn((5, w.L), device=dev).to(torch.bfloat16)
    recv_e = torch.tensor([0, 3, E_loc, 7, 1], dtype=torch.int32, device=dev)  # row 2 out of range
    y, ss = s.experts(recv_z, recv_e)
    torch.cuda.synchronize()
    code, _ = moe.last_device_status(s.config(1, s.ws_experts))
    assert moe.STATUS[code] == "MUSE_ERR_DEVICE"
    assert torch.count_nonzero(y[2]) == 0 and torch.count_nonzero(ss[2]) == 0
    assert torch.count_nonzero(y[0]) > 0 and torch.count_nonzero(y[4]) > 0


# --------------------------------------------------------------------- host-only checks
def _tiny_weights(E_loc):
    w = W.WORKLOADS["tiny"]
    inp = W.make_inputs(w, "cpu", names=["W_router", "W_pool", "W_gate", "W_up", "W_down", "gamma", "W_unpool"])
    for n in ("W_gate", "W_up", "W_down"):
        inp[n] = inp[n][:E_loc].contiguous()
    return w, inp


def test_expert_shard_rejects_a_split_that_does_not_divide_or_match():
    from latent_mixture_experts_moe_b200 import ep
    w, inp = _tiny_weights(4)
    with pytest.raises(ValueError, match="do not split"):
        ep.ExpertShard(inp, 0, 3, T_max=16, k=w.k)          # 8 experts over 3 ranks
    with pytest.raises(ValueError, match="this rank owns"):
        ep.ExpertShard(inp, 0, 4, T_max=16, k=w.k)          # holds 4, owns 2


def test_expert_shard_sizes_its_buffers_for_the_worst_case_receive():
    from latent_mixture_experts_moe_b200 import ep
    import latent_mixture_experts_moe_b200 as moe
    w, inp = _tiny_weights(4)
    s = ep.ExpertShard(inp, 1, 2, T_max=16, k=w.k)
    assert s.rows_max == 2 * 16 * min(w.k, 4)
    assert s.send_z.shape == (16 * w.k, w.L) and s.send_expert.shape == (16 * w.k,)
    cfg = s.config(16)
    assert s.ws_home.numel() == moe.ep_workspace_layout(cfg, 2, moe.EP_HOME)["total"]
    assert s.ws_experts.numel() == moe.ep_workspace_layout(cfg, 2, moe.EP_EXPERTS, s.rows_max)["total"]
    assert int(s.ws_home.abs().sum()) == 0 and int(s.ws_experts.abs().sum()) == 0  # start zeroed
    assert s.gamma_local.shape == (4, w.L)
    assert torch.equal(s.gamma_local, inp["gamma"][4:8])   # rank 1's experts 4..7
    # a rank with no tokens sends nothing and never calls the library
    z, e, counts = s.dispatch(torch.empty((0, w.D)))
    assert z.shape[0] == 0 and e.shape[0] == 0 and counts == [0, 0]
