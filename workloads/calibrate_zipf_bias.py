"""Writes the stored selection bias of the Zipf-skewed prefill workload.

The skewed prefill workload (T=8192 tokens, E=256 experts, top-8) wants expert
popularity to follow Zipf with exponent 1.2. A per-expert bias that only changes which
experts are selected -- the "e_score_correction_bias" of the Muse Spark Open deep dive,
§4.2 -- is tuned on the workload's own seeded tokens with the sign rule the same
section gives for load balancing (b_i moves by a step gamma towards the target count,
minus the mean step), here steering towards the water-filled Zipf targets of
workloads.zipf_target_loads instead of the mean load.

It calls only the FP64 oracle for the routing (router logits and top-k); its output is
a plain text file of 256 float32 values that both the CUDA path and the oracle read.

    python -m workloads.calibrate_zipf_bias
"""
from __future__ import annotations

import sys

import numpy as np
import torch

import oracle
import workloads as W


def calibrate(w: W.Workload, iters: int = 400, step0: float = 0.05, step1: float = 2e-4,
              verbose: bool = True) -> np.ndarray:
    x = oracle.as_f64(W.make_tensor(w, "x"))
    wr = oracle.as_f64(W.make_tensor(w, "W_router"))
    logits = oracle.router_logits(x, wr)
    target_by_rank = W.zipf_target_loads(w.T, w.E, w.k).numpy()
    expert_of_rank = W.zipf_rank_to_expert(w).numpy()
    target = np.empty(w.E)
    target[expert_of_rank] = target_by_rank
    b = np.zeros(w.E, dtype=np.float32)
    best, best_err = b.copy(), np.inf
    for it in range(iters):
        step = step0 * (step1 / step0) ** (it / max(1, iters - 1))
        idx = oracle.select_topk(logits + b.astype(np.float64)[None, :], w.k)
        n = np.bincount(idx.ravel(), minlength=w.E).astype(np.float64)
        err = np.abs(n - target).sum() / (w.T * w.k)
        if err < best_err:
            best, best_err = b.copy(), err
        delta = step * np.sign(target - n)
        b = (b + (delta - delta.mean())).astype(np.float32)
        if verbose and it % 50 == 0:
            print(f"iter {it:4d} step {step:.2e} L1 share error {err:.4f}", flush=True)
    if verbose:
        print(f"best L1 share error {best_err:.4f}")
    return best


def main(argv=None) -> int:
    w = W.WORKLOADS["prefill_zipf"]
    b = calibrate(w)
    path = W.zipf_bias_path(w)
    with open(path, "w") as f:
        f.write("# Selection-only router bias of the Zipf(s=1.2) skewed prefill workload,\n")
        f.write(f"# T={w.T} D={w.D} E={w.E} k={w.k} seed={w.seed}; written by workloads/calibrate_zipf_bias.py\n")
        f.write("# expert  bias(float32)\n")
        for e, v in enumerate(b):
            f.write(f"{e} {float(v)!r}\n")
    print("wrote", path)
    return 0


if __name__ == "__main__":
    sys.exit(main(sys.argv[1:]))
