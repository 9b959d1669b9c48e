"""The allocation-free forward entry point, muse_latent_moe_forward_static_scratch.

Some callers cannot allocate device memory at all: a plug-in whose host application
owns every allocation, code that runs where cudaMalloc is not permitted or would stall
the device, a service with a fixed memory budget. This entry point serves them by taking
its workspace from a scratch array built into the library instead of from the caller.
These tests call it through the C ABI and check that it gives the same block output as
the regular entry point (muse_latent_moe_forward with a caller-owned workspace), on two
calls in a row, and that sizes beyond the array are refused before any launch.

This file is collected last on purpose, so a stop-at-first-failure run has already run
every other test when it gets here.
"""
import ctypes

import pytest
import torch

import latent_mixture_experts_moe_b200 as moe
import workloads as W


def _weights(inp):
    return [inp[n] for n in ("W_router", "W_pool", "W_gate", "W_up", "W_down", "gamma", "W_unpool")]


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["tiny", "mid"])
def test_static_scratch_forward_matches_workspace_forward_on_two_calls(name):
    """Same kernels, same sizes: the output equals the regular entry point's bit for bit,
    on two calls in a row with different tokens; the status word of the built-in array
    (read with a config that names no workspace) reports success; and a call after the
    first allocates no device memory (free memory unchanged across it)."""
    w = W.WORKLOADS[name]
    inp = W.make_inputs(w, "cuda")
    x2 = torch.empty_like(inp["x"])
    W.fill(x2, w.seed, W.TID["x"], 1.0, start=w.T * w.D)          # a second batch of tokens
    model = moe.LatentMoE({k: v for k, v in inp.items() if k != "x"}, T_max=w.T, k=w.k, eps=w.eps)
    cfg = model.config(w.T)                                       # no workspace given
    assert moe.workspace_size(cfg) <= moe.STATIC_SCRATCH_BYTES
    for call, x in enumerate((inp["x"], x2)):
        ref = model(x)                                            # regular entry point
        out = torch.full_like(ref, float("nan"))
        torch.cuda.synchronize()
        free0 = torch.cuda.mem_get_info()[0]
        moe.forward_static_scratch(cfg, x, *_weights(inp), out)
        torch.cuda.synchronize()
        free1 = torch.cuda.mem_get_info()[0]
        assert torch.equal(out, ref), f"{name}: static-scratch call {call} differs"
        code, detail = moe.last_device_status(cfg)                # cfg.workspace is NULL
        assert code == 0, (moe.STATUS.get(code), hex(detail))
        if call > 0:                                              # kernels loaded by the first
            assert free1 == free0, f"device memory changed by {free0 - free1} bytes"


def test_static_scratch_rejects_sizes_beyond_the_array():
    # the full prefill layer needs far more than the built-in array: refused up front,
    # before any CUDA call (this check runs without a GPU)
    w = W.WORKLOADS["prefill"]
    cfg = moe.make_config(w.T, w.D, w.L, w.I, w.E, w.k, w.dtype, w.eps)
    assert moe.workspace_size(cfg) > moe.STATIC_SCRATCH_BYTES
    ptrs = [ctypes.c_void_p(4096 * (i + 1)) for i in range(9)]
    code = moe.lib().muse_latent_moe_forward_static_scratch(ctypes.byref(cfg), *ptrs, None)
    assert code == 3, moe.STATUS.get(code)
