"""The N > 1 path of bench.py, on CPU with gloo (world size 2): each rank is a replica
with its own slice of one seeded token stream (no data-path exchange), the timing is the
max over ranks, and the block computed per shard equals the block on the whole batch
(tokens are independent), checked with the FP64 oracle."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import oracle
        import workloads as W
        w = W.WORKLOADS["tiny"]
        dev = torch.device("cpu")
        # replica shard of the token stream
        x = bench.rank_tokens(w, rank, dev)
        shards = [torch.empty_like(x) for _ in range(world)]
        dist.all_gather(shards, x)
        # max over ranks of the timing, barrier
        bench.barrier(world)
        tmax = bench.all_max(1.5 + rank, world, dev)
        # each rank runs the block on its shard; rank 0 compares with the whole batch
        inp = W.make_inputs(w, "cpu", names=["W_router", "W_pool", "W_gate", "W_up", "W_down", "gamma",
                                              "W_unpool"])
        f = oracle.as_f64
        def block(xx):
            return oracle.latent_moe_forward(f(xx), f(inp["W_router"]), f(inp["W_pool"]),
                                             (f(inp["W_gate"]), f(inp["W_up"]), f(inp["W_down"])), f(inp["gamma"]),
                                             f(inp["W_unpool"]), w.k, w.eps)["out"]
        out = torch.from_numpy(block(x))
        outs = [torch.empty_like(out) for _ in range(world)]
        dist.all_gather(outs, out)
        if rank == 0:
            whole = torch.empty((world * w.T, w.D), dtype=x.dtype)
            W.fill(whole, w.seed, W.TID["x"], 1.0)
            ref = block(whole)
            q.put(dict(stream_ok=bool(torch.equal(torch.cat(shards), whole)), tmax=tmax,
                       block_err=float(np.abs(torch.cat(outs).numpy() - ref).max())))
    finally:
        dist.destroy_process_group()


def test_two_replicas_partition_one_token_stream_and_agree_with_the_whole_batch():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = q.get(timeout=300)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert res["stream_ok"]
    assert res["tmax"] == 2.5
    assert res["block_err"] < 1e-12


def test_job_throughput_counts_every_rank():
    import bench
    assert bench.job_tokens_per_s(1, 8192, 10, 100.0) == 8192 * 10 / 0.1
    assert bench.job_tokens_per_s(4, 8192, 10, 100.0) == 4 * 8192 * 10 / 0.1
