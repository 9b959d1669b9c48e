"""The seeded input generator shared by the oracle and the CUDA path (CPU): SplitMix64 as
published, slab and chunk invariance, the Box-Muller normals' range and moments, and the
Zipf load targets."""
import math

import numpy as np
import pytest
import torch

import workloads as W

M64 = (1 << 64) - 1


def splitmix64_finalise(z: int) -> int:
    """The SplitMix64 output function (Steele, Lea and Flood, "Fast splittable pseudorandom
    number generators", OOPSLA 2014; the constants of the public-domain C reference)."""
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9 & M64
    z = (z ^ (z >> 27)) * 0x94D049BB133111EB & M64
    return z ^ (z >> 31)


def test_hash_is_splitmix64_of_the_golden_ratio_counter():
    rng = np.random.default_rng(0)
    seeds = [0, 1, 12345] + [int(s) for s in rng.integers(0, 2**31, 3)]
    for seed in seeds:
        for tid in (1, 4, 15):
            got = W.uniform_u64(seed, tid, 16)
            base = (seed * 0x9E3779B97F4A7C15 + tid * 0xD1B54A32D192ED03) & M64
            for i in range(16):
                ctr = (2 * i + base) & M64
                want = splitmix64_finalise(ctr * 0x9E3779B97F4A7C15 & M64)
                assert int(got[i]) & M64 == want, (seed, tid, i)


def test_expert_slab_equals_the_slice_of_the_whole_tensor():
    w = W.WORKLOADS["tiny"]
    for name in ("W_gate", "W_up", "W_down"):
        whole = W.make_tensor(w, name)
        for e in (0, 3, w.E - 1):
            assert torch.equal(W.expert_slab(w, name, e), whole[e])


def test_fill_does_not_depend_on_the_chunk_size_or_the_start_split():
    a = torch.empty(1000, dtype=torch.float64)
    b = torch.empty(1000, dtype=torch.float64)
    W.fill(a, 7, 3, 1.0)
    W.fill(b, 7, 3, 1.0, chunk=37)
    assert torch.equal(a, b)
    c = torch.empty(600, dtype=torch.float64)
    W.fill(c, 7, 3, 1.0, start=400)
    assert torch.equal(c, a[400:])


def test_normals_are_finite_and_standard():
    x = W.normal_f64(0, 1, 0, 1 << 20)
    assert torch.isfinite(x).all()
    n = x.numel()
    mean, var = float(x.mean()), float(x.var())
    assert abs(mean) < 5 / math.sqrt(n)
    assert abs(var - 1) < 5 * math.sqrt(2 / n)
    # tail mass beyond 3 sigma: 0.0027 for a standard normal
    tail = float((x.abs() > 3).double().mean())
    assert abs(tail - 0.0026998) < 5 * math.sqrt(0.0027 / n)
    # different tensor ids give different streams
    assert not torch.equal(W.normal_f64(0, 1, 0, 64), W.normal_f64(0, 2, 0, 64))


@pytest.mark.parametrize("T,E,k", [(8192, 256, 8), (512, 64, 4), (64, 16, 2)])
def test_zipf_targets_are_feasible_and_ordered(T, E, k):
    n = W.zipf_target_loads(T, E, k)
    assert n.shape == (E,)
    assert abs(float(n.sum()) - T * k) < 1e-6 * T * k
    assert float(n.max()) <= T + 1e-9
    assert bool((n[:-1] >= n[1:] - 1e-9).all())          # rank order: non-increasing


def test_stored_zipf_bias_matches_its_workload():
    w = W.WORKLOADS["prefill_zipf"]
    b = W.zipf_router_bias(w)
    assert b.shape == (w.E,) and b.dtype == torch.float32 and bool(torch.isfinite(b).all())
    perm = W.zipf_rank_to_expert(w)
    assert sorted(perm.tolist()) == list(range(w.E))
