"""The algorithmic FLOPs and bytes bench.py divides by measured time (its roofline
numerators), checked against the per-token accounting the pages print and against the sum
of the per-kernel figures. Host arithmetic only."""
import pytest

import bench
import workloads as W
from golden_io import lines


def golden_accounting():
    return {s.split()[0]: float(s.split()[1]) for s in lines("accounting.txt")}


def test_step_flops_per_token_equal_the_printed_moe_flops():
    """943.7 MFLOP per token per layer ("Muse Spark Open deep dive" §4.3 table): 2 x the
    active parameters (router, pooler, k experts, unpooler)."""
    g = golden_accounting()
    for name in ("prefill", "decode"):
        w = W.WORKLOADS[name]
        flops, _, fp4 = bench.step_work(w, n_touched=w.E)
        assert fp4 == 0
        assert abs(flops / w.T / 1e6 - g["moe_mflops_per_token_printed"]) < 0.05
        # the printed active count includes the two L-wide norm gains (router + projections +
        # norms = 69,214,208), which carry no multiply-accumulate
        assert flops / w.T == 2 * (g["params_active_per_token"] - 2 * w.L)


@pytest.mark.parametrize("name,n_touched,gflop,gbytes", [
    ("prefill", 256, 7731, 26.18),   # every expert touched
    ("decode", 222, 60.4, 22.48),    # about 222 distinct experts under uniform routing
])
def test_step_work_matches_the_config_table(name, n_touched, gflop, gbytes):
    """The layer's algorithmic work: x and out, the router / pooler / unpooler weights, and
    each distinct touched expert's weights once (bf16)."""
    w = W.WORKLOADS[name]
    flops, byts, _ = bench.step_work(w, n_touched)
    assert abs(flops / 1e9 - gflop) / gflop < 0.002
    assert abs(byts / 1e9 - gbytes) / gbytes < 0.005


@pytest.mark.parametrize("name", ["prefill", "decode", "nvfp4", "nvfp4_w4a4", "mid", "tiny"])
def test_kernel_flops_add_up_to_the_step(name):
    w = W.WORKLOADS[name]
    n = min(w.E, w.T * w.k)
    work = bench.stage_work(w, n)
    step_flops, _, fp4 = bench.step_work(w, n)
    assert sum(f for f, _ in work.values()) == step_flops
    if w.act == "nvfp4":
        assert fp4 == work["gate_up_swiglu"][0] + work["down_sumsq"][0]


def test_grouped_gemm_bytes_are_weights_once_plus_rows_once():
    """Gate/up at prefill: every expert's gate and up weights once (17.18 GB) plus the
    gathered latent rows read and h written once (0.54 GB each) -- the figure the DRAM
    traffic of the kernel is compared with. W4A4: weights at 0.5625 B, latent rows read as
    codes (0.5625 B per value), h written in bf16."""
    w = W.WORKLOADS["prefill"]
    _, b = bench.stage_work(w, 256)["gate_up_swiglu"]
    A = w.T * w.k
    assert b == 256 * 2 * w.I * w.L * 2 + A * w.L * 2 + A * w.I * 2
    assert abs(b / 1e9 - 18.25) < 0.01
    q = W.WORKLOADS["nvfp4_w4a4"]
    _, bq = bench.stage_work(q, 256)["gate_up_swiglu"]
    Aq = q.T * q.k
    assert bq == 256 * 2 * q.I * q.L * 0.5625 + Aq * q.L * 0.5625 + Aq * q.I * 2
