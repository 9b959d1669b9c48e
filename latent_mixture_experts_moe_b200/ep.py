"""Expert parallelism (EP) for the latent-MoE block over G ranks.

Rank r owns experts [r * E / G, (r + 1) * E / G) and replicates the router, pooler,
unpooler and every expert's gain (Muse Spark Open deep dive, §4.3, implementation notes:
expert tensors split along the expert dimension, tokens moved by an EP dispatch, norm
weights replicated; on the expert side each received row has one expert and unit weight,
and the routing weights are applied after the rows come back, keeping the per-expert norm
ahead of the weighting). What crosses between GPUs is the 4096-wide latent, one row per
(token, expert) pair, and its expert output plus L/32 partial sums of squares coming back.

One forward is three library calls around two all-to-all exchanges:

    send = dispatch(x)            routing, pooler, send buffer grouped by rank
    recv = all_to_all(send)       rows for this rank's experts, from every rank
    ret  = experts(recv)          gate/up + SwiGLU, down, sums of squares
    back = all_to_all(ret)        each rank's results back into its send rows
    out  = combine(x, back)       per-expert norm, weighted combine, unpooler

The exchanges use torch.distributed (NCCL over NVLink on GPUs); the row counts are read on
the host to size them, the one synchronisation of the step. Everything else here is
argument marshalling: every step of the block runs in the library's kernels.
"""
from __future__ import annotations

from typing import Dict, List, Optional, Sequence, Tuple

from . import (EP_EXPERTS, EP_HOME, _ptr, block_config, ep_combine, ep_dispatch, ep_experts, ep_workspace_layout,
               expert_operands, expert_weight_dims)


class ExpertShard:
    """One rank's part of the block under expert parallelism.

    weights: W_router [E, D], W_pool [L, D], gamma [E, L] (every expert's gain, or the
    shared [L]), W_unpool [D, L] and the optional router_bias / gains, as for LatentMoE;
    the expert matrices hold only this rank's E / G experts: W_gate / W_up [E/G, I, L],
    W_down [E/G, L, I] (or their NVFP4 codes, scales and matrix scales).
    T_max: most tokens per call on this rank. rows_max: most rows one call receives
    (default G * T_max * min(k, E / G), the bound when every rank sends T_max tokens).
    """

    def __init__(self, weights: Dict, ep_rank: int, ep_size: int, T_max: int, k: int, eps: float = 1e-6,
                 rows_max: Optional[int] = None, **modes):
        import torch
        E, D = weights["W_router"].shape
        if E % ep_size:
            raise ValueError(f"E={E} experts do not split over {ep_size} ranks")
        self.E_loc = E // ep_size
        I, L, self.nvfp4 = expert_weight_dims(weights)
        lead = (weights["W_gate_codes"] if self.nvfp4 else weights["W_gate"]).shape[0]
        if lead != self.E_loc:
            raise ValueError(f"expert tensors hold {lead} experts, this rank owns {self.E_loc}")
        self.w = dict(weights)
        self.experts_args = expert_operands(weights, self.nvfp4)
        self.rank, self.G, self.T_max, self.k = ep_rank, ep_size, T_max, k
        self.dtype = {torch.float32: "f32", torch.bfloat16: "bf16"}[weights["W_router"].dtype]
        self.act = weights["W_router"].dtype
        self.dims = dict(D=int(D), L=L, I=I, E=int(E), k=k, eps=eps)
        self.modes = modes
        dev = weights["W_router"].device
        self.rows_max = rows_max if rows_max is not None else ep_size * T_max * min(k, self.E_loc)
        home = ep_workspace_layout(self.config(T_max), ep_size, EP_HOME)["total"]
        shard = ep_workspace_layout(self.config(T_max), ep_size, EP_EXPERTS, max(self.rows_max, 1))["total"]
        # zeroed once, so that a status read before a side has run (a rank with no tokens, a
        # shard that received no rows) reads MUSE_OK
        self.ws_home = torch.zeros(home, dtype=torch.uint8, device=dev)
        self.ws_experts = torch.zeros(shard, dtype=torch.uint8, device=dev)
        self.send_z = torch.empty((T_max * k, L), dtype=self.act, device=dev)
        self.send_expert = torch.empty(T_max * k, dtype=torch.int32, device=dev)
        self.rank_counts = torch.empty(ep_size, dtype=torch.int32, device=dev)
        # the local experts' gains, read by the down projection in input-scaled norm mode
        g = weights["gamma"]
        self.gamma_local = g if g.dim() == 1 else g[ep_rank * self.E_loc:(ep_rank + 1) * self.E_loc].contiguous()

    def config(self, T: int, workspace=None):
        return block_config(T, self.dims, self.dtype, self.modes, self.w, self.nvfp4, workspace)

    def dispatch(self, x, topk_idx=None, topk_w=None, stream=None) -> Tuple[object, object, List[int]]:
        """Routing, pooler and send buffer for this rank's tokens x [T, D]: (send_z [T*k, L],
        send_expert [T*k] int32, rows per destination rank). Synchronises the stream to read
        the counts; a rank with no tokens sends nothing."""
        import torch
        T = x.shape[0]
        if T > self.T_max:
            raise ValueError(f"T={T} exceeds T_max={self.T_max}")
        n = T * self.k
        if T == 0:
            return self.send_z[:0], self.send_expert[:0], [0] * self.G
        cfg = self.config(T, self.ws_home)
        cfg.topk_idx_out, cfg.topk_w_out = _ptr(topk_idx), _ptr(topk_w)
        ep_dispatch(cfg, self.G, x, self.w["W_router"], self.w["W_pool"], self.send_z, self.send_expert,
                    self.rank_counts, stream)
        (stream if stream is not None else torch.cuda.current_stream()).synchronize()
        return self.send_z[:n], self.send_expert[:n], self.rank_counts.tolist()

    def experts(self, recv_z, recv_expert, stream=None):
        """This rank's experts over the received rows: (ret_y [R, L], ret_ss float [R, L/32])."""
        import torch
        R = recv_z.shape[0]
        if R > self.rows_max:
            raise ValueError(f"{R} rows received, the expert workspace holds {self.rows_max}")
        L = self.dims["L"]
        ret_y = torch.empty((R, L), dtype=self.act, device=recv_z.device)
        ret_ss = torch.empty((R, L // 32), dtype=torch.float32, device=recv_z.device)
        cfg = self.config(self.T_max, self.ws_experts)
        wg, wu, wd = self.experts_args
        ep_experts(cfg, self.G, R, recv_z, recv_expert, wg, wu, wd, self.gamma_local, ret_y, ret_ss, stream)
        return ret_y, ret_ss

    def combine(self, x, back_y, back_ss, out=None, stream=None):
        """Per-expert norm, weighted combine and unpooler of this rank's tokens, from the rows
        of its send buffer that came back (the same workspace as the preceding dispatch)."""
        import torch
        T = x.shape[0]
        if out is None:
            out = torch.empty((T, self.dims["D"]), dtype=x.dtype, device=x.device)
        if T == 0:
            return out
        cfg = self.config(T, self.ws_home)
        ep_combine(cfg, self.G, x, back_y, back_ss, self.w["gamma"], self.w["W_unpool"], out, stream)
        return out


def exchange_counts(send_counts: Sequence[int], device, group=None) -> List[int]:
    """All-to-all of the per-rank row counts: element q of the result is what rank q sends here."""
    import torch
    import torch.distributed as dist
    s = torch.tensor(list(send_counts), dtype=torch.int64, device=device)
    r = torch.empty_like(s)
    dist.all_to_all_single(r, s, group=group)
    return r.tolist()


def exchange_rows(t, send_counts: Sequence[int], recv_counts: Sequence[int], group=None):
    """All-to-all of row blocks: rows [sum(send_counts[:q]), + send_counts[q]) of t go to rank
    q; the result holds the blocks received, in source rank order."""
    import torch.distributed as dist
    out = t.new_empty((int(sum(recv_counts)),) + tuple(t.shape[1:]))
    dist.all_to_all_single(out, t.contiguous(), output_split_sizes=list(recv_counts),
                           input_split_sizes=list(send_counts), group=group)
    return out


def ep_forward(shard, x, group=None):
    """One expert-parallel forward of this rank's tokens x; every rank of `group` calls it
    at the same time with its own shard and tokens (any number of tokens, zero included).
    shard: an ExpertShard, or any object with the same dispatch / experts / combine."""
    send_z, send_expert, send_counts = shard.dispatch(x)
    recv_counts = exchange_counts(send_counts, x.device, group)
    recv_z = exchange_rows(send_z, send_counts, recv_counts, group)
    recv_expert = exchange_rows(send_expert, send_counts, recv_counts, group)
    ret_y, ret_ss = shard.experts(recv_z, recv_expert)
    back_y = exchange_rows(ret_y, recv_counts, send_counts, group)
    back_ss = exchange_rows(ret_ss, recv_counts, send_counts, group)
    return shard.combine(x, back_y, back_ss)


def ep_forward_one_device(shards: Sequence, xs: Sequence):
    """The same forward for all G ranks' shards held on one device, the two exchanges done
    by slicing and concatenating on the host's order of calls (no kernel waits on another):
    for validating an EP configuration on one GPU. Returns every rank's output."""
    import torch
    G = len(shards)
    sends = [s.dispatch(x) for s, x in zip(shards, xs)]
    starts = [[sum(c[:q]) for q in range(G)] for _, _, c in sends]

    def block(q, r, t):  # rows rank q sends to rank r
        return t[starts[q][r]:starts[q][r] + sends[q][2][r]]

    rets = []
    for r in range(G):
        recv_z = torch.cat([block(q, r, sends[q][0]) for q in range(G)])
        recv_e = torch.cat([block(q, r, sends[q][1]) for q in range(G)])
        rets.append(shards[r].experts(recv_z, recv_e))
    outs = []
    for q in range(G):
        # rank r's results for rank q's rows sit after the rows r received from ranks < q
        back_y, back_ss = [], []
        for r in range(G):
            lo = sum(sends[p][2][r] for p in range(q))
            n = sends[q][2][r]
            back_y.append(rets[r][0][lo:lo + n])
            back_ss.append(rets[r][1][lo:lo + n])
        outs.append(shards[q].combine(xs[q], torch.cat(back_y), torch.cat(back_ss)))
    return outs
