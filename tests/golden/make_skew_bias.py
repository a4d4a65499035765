"""Write the stored selection biases of the skewed-routing workloads (skew_bias_*.txt).

The skewed workload asks for expert popularity that follows Zipf(1.1) over a seeded random
permutation of the experts, with some experts that receive no token.  The pages never mention a
router bias; the reading taken here is the DeepSeek-V3 scheme the pages name, a per-expert bias added
to the sigmoid scores for selection only, and that bias shapes the load.

Recipe (uses only the CPU oracle and the seeded input generator):
  1. draw a separate calibration batch x_cal (seed offset 77, T_cal tokens) and the workload's W_r;
  2. compute the oracle's sigmoid scores once;
  3. target count of the expert at popularity rank r (1-based): T_cal*k * r^-1.1 / sum, capped at
     0.97*T_cal (an expert can take each token once);
  4. repeat n_rounds: route with the current bias (oracle.select), then
     b_e += eta * (ln(target_e + 0.5) - ln(observed_e + 0.5)), eta = 0.05;
  5. set b = -4 on the n_zero lowest-ranked experts (their selection value drops below every
     other expert's, so they receive no token);
  6. write the bias (fp32, one value per expert) with this recipe and the realised load in the
     header.

Run:  python tests/golden/make_skew_bias.py
"""
from __future__ import annotations

import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import beam_synth as bs  # noqa: E402
import oracle  # noqa: E402

HERE = os.path.dirname(os.path.abspath(__file__))


def calibrate(wl: bs.Workload, T_cal: int, n_zero: int, n_rounds: int = 60, eta: float = 0.05, zipf_s: float = 1.1):
    E, k = wl.n_experts, wl.topk
    x = bs.make_x(wl, T=T_cal, seed_offset=77)
    W = bs.make_router(wl).numpy()
    score = oracle.router_scores(oracle.bf16_bits(x), W)
    g = torch.Generator().manual_seed(bs.sub_seed(wl.seed, "perm"))
    perm = torch.randperm(E, generator=g).numpy()        # perm[r] = expert at popularity rank r
    rank = np.empty(E, dtype=np.int64)
    rank[perm] = np.arange(E)
    p = (rank + 1.0) ** (-zipf_s)
    p /= p.sum()
    target = np.minimum(T_cal * k * p, 0.97 * T_cal)
    b = np.zeros(E, dtype=np.float64)
    for _ in range(n_rounds):
        r = oracle.select(score, wl.layer, b.astype(np.float32))
        obs = np.bincount(r["ids"].ravel(), minlength=E)
        b += eta * (np.log(target + 0.5) - np.log(obs + 0.5))
    b[rank >= E - n_zero] = -4.0
    b = b.astype(np.float32)
    r = oracle.select(score, wl.layer, b)
    obs = np.bincount(r["ids"].ravel(), minlength=E)
    return b, obs, target, perm


def write(path: str, wl: bs.Workload, T_cal: int, n_zero: int, b, obs, perm):
    mean = T_cal * wl.topk / wl.n_experts
    with open(path, "w") as f:
        f.write(f"# Selection bias for workload '{wl.name}' (E={wl.n_experts}, G={wl.n_groups}, "
                f"keep {wl.topk_groups}, top-{wl.topk}, seed {wl.seed}).\n")
        f.write("# Written by tests/golden/make_skew_bias.py (CPU oracle routing on a separate calibration draw).\n")
        f.write(f"# Target: Zipf(1.1) popularity over a seeded expert permutation; {n_zero} lowest-ranked experts "
                f"biased to -4.\n")
        f.write(f"# Calibration draw T={T_cal}: max/mean load {obs.max() / mean:.2f}, "
                f"experts with 0 tokens: {int((obs == 0).sum())}, top-5 loads {sorted(obs.tolist())[-5:][::-1]}.\n")
        f.write(f"# Most popular experts (rank order): {perm[:8].tolist()}\n")
        for i in range(0, len(b), 8):
            f.write(" ".join(f"{v:.9g}" for v in b[i:i + 8]) + "\n")


def main():
    for wl, T_cal, n_zero, fname in ((bs.WORKLOADS["skew"], 4096, 8, "skew_bias_beam.txt"),
                                     (bs.PARITY_CASES["mid_skew"], 2048, 4, "skew_bias_mid.txt")):
        b, obs, target, perm = calibrate(wl, T_cal, n_zero)
        path = os.path.join(HERE, fname)
        write(path, wl, T_cal, n_zero, b, obs, perm)
        mean = T_cal * wl.topk / wl.n_experts
        print(f"{fname}: max/mean {obs.max() / mean:.2f}, zero-load experts {(obs == 0).sum()}, "
              f"top loads {sorted(obs.tolist())[-5:][::-1]}")


if __name__ == "__main__":
    main()
