"""Comparison rules between the CUDA path and the CPU oracle.

- integer accumulators, activation codes and routing indices: bit-exact;
- routing: a token's expert list may differ from the oracle's only where the
  oracle's own selection scores are within 1e-6 relative (slot j of the GPU
  list must have an oracle score within that bound of the oracle's slot j);
  such tokens are counted, reported and left out of downstream comparisons;
- requantised h codes: within +-1, on at most 0.1% of entries;
- final fp32 outputs: relative L2 error <= 2e-3.
"""
from __future__ import annotations

import numpy as np

NEAR_TIE_REL = 1e-6
HQ_MAX_FRAC = 1e-3
OUT_REL_L2 = 2e-3


def routing_mismatches(gpu_idx, orc_idx, orc_sel, rel: float = NEAR_TIE_REL):
    """Returns (allowed_tokens, bad_tokens): tokens whose GPU routing differs
    from the oracle's within the near-tie rule, and tokens that break it."""
    gpu_idx = np.asarray(gpu_idx)
    orc_idx = np.asarray(orc_idx)
    sel = np.asarray(orc_sel, np.float64)
    allowed, bad = [], []
    for t in range(orc_idx.shape[0]):
        g, o = gpu_idx[t], orc_idx[t]
        if np.array_equal(g, o):
            continue
        ok = len(set(g.tolist())) == len(g) and all(0 <= e < sel.shape[1] for e in g)
        if ok:
            for j in range(len(o)):
                if abs(sel[t, g[j]] - sel[t, o[j]]) > rel * abs(sel[t, o[j]]):
                    ok = False
                    break
        (allowed if ok else bad).append(t)
    return allowed, bad


def rel_l2(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / den) if den > 0 else float(np.linalg.norm(a))


def hq_close(gpu_hq, orc_hq) -> tuple:
    """(max |diff|, fraction of entries that differ)."""
    d = np.abs(np.asarray(gpu_hq, np.int32) - np.asarray(orc_hq, np.int32))
    return int(d.max()) if d.size else 0, float((d != 0).mean()) if d.size else 0.0
