"""Derive the Zipf amplitude beta of the skewed-routing workload with the oracle.

The skewed workload's router bias is uniform(-0.01, 0.01) plus
beta * (rank_e + 1) ** -1.1 over a seeded ranking of the 256 experts, with beta
chosen so that on layer 0's draws (64 bf16 tokens, parameter-free RMSNorm, the
oracle's router) the 16 most-assigned experts take 70% of the 64 * 8
assignments.  This script bisects beta with the CPU oracle only and writes the
value to tests/golden/zipf_beta.json; workloads.ZIPF_BETA_SKEWED carries it.

    python tests/golden/calibrate_zipf_beta.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle as O  # noqa: E402
import workloads as W  # noqa: E402

TARGET, TOL = 0.70, 0.02


def top16_share(wl, seed, beta, x_in, w_router):
    bias = W.router_bias(wl, seed, 0, zipf_beta=beta)
    idx, _ = O.route(x_in, w_router, bias, wl.top_k, wl.routed_scale)
    counts = np.bincount(idx.reshape(-1), minlength=wl.n_experts)
    return np.sort(counts)[::-1][:16].sum() / idx.size


def calibrate(seed=0):
    wl = W.workload(4)
    x0 = W.tokens(wl, seed).float().numpy().astype(np.float64)
    x_in = O.rmsnorm(x0)
    wr = W.router_weight(wl, seed, 0)
    lo, hi = 0.0, 4.0
    assert top16_share(wl, seed, hi, x_in, wr) > TARGET
    for _ in range(40):
        mid = 0.5 * (lo + hi)
        if top16_share(wl, seed, mid, x_in, wr) < TARGET:
            lo = mid
        else:
            hi = mid
    beta = float(np.float32(hi))
    share = top16_share(wl, seed, beta, x_in, wr)
    assert abs(share - TARGET) <= TOL, share
    return beta, share


if __name__ == "__main__":
    beta, share = calibrate()
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "zipf_beta.json")
    with open(out, "w") as fh:
        json.dump({"zipf_beta": beta, "top16_share": share, "seed": 0,
                   "written_by": "tests/golden/calibrate_zipf_beta.py (CPU oracle only)"}, fh, indent=1)
    print(beta, share)
