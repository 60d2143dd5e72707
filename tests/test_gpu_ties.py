"""Exact ties in the router select the lower expert index, on every router
implementation of the library, and the ABI's expert range up to E = 1024 runs.

The router is DeepSeek-V3 style (takumi3488 article, teacher-forcing section):
experts are chosen by sigmoid score plus selection bias, and when two
selection values are equal the lower expert index takes the slot.  Random
inputs almost never tie exactly, so the inputs here are built to tie:

- "zero": an all-zero router matrix, so every logit is exactly 0 and every
  score exactly 0.5 on both sides; the biases are multiples of 0.125 on a few
  levels, each level shared by more than k experts spread over the index range
  by a seeded permutation.  The selection value 0.5 + bias is exact, the top
  level ties for every slot, and the k lowest indices on it must win, in
  ascending order.
- "dup": experts in groups of three share one router row and one bias (group
  members spread over the index range), so a group's selection values are
  bit-equal on each side (each side computes every row with the same
  arithmetic).  k is not a multiple of 3, so the k-th slot always falls inside
  a tied group: the group's lower indices must take it.

Here the comparison is exact: no near-tie allowance (the oracle's tied values
are bit-equal, and so are the GPU's).  The router implementations covered:
the single-launch decode kernel (E <= 256 register top-k; E > 256 shared-memory
top-k), the small-T router GEMV with its last-CTA top-k, the tiled router with
the register top-k and in-kernel bucketing (E <= 256) or the shared-memory
top-k and the separate bucketing kernel (E > 256), and the allocation-free
router.  The layer cases also run E = 512 and 1024 end to end on the decode,
dp4a multi-kernel and tensor-core paths against the oracle.
"""
import numpy as np
import pytest
import torch

import expert_ffn_router_b200 as M
import oracle as O
import workloads as W
from parity_utils import OUT_REL_L2, rel_l2

pytestmark = pytest.mark.gpu

TIE_TAG = 0x71E5


def tie_router(E: int, d: int, k: int, kind: str, seed: int = 0):
    """Router weights [E][d] and bias [E] (fp32) whose selection values tie."""
    key = W.stream_key(seed, TIE_TAG, E, d, k, 1 if kind == "zero" else 2)
    perm = W.permutation(key, E)
    if kind == "zero":
        levels = max(2, E // (k + 1))  # every level holds more than k experts
        wr = torch.zeros(E, d, dtype=torch.float32)
        bias = (((perm % levels) - levels // 2).to(torch.float64) * 0.125).to(torch.float32)
        return wr, bias
    # the experts whose permuted positions are 3g, 3g+1, 3g+2 form group g; the
    # E % 3 left over get rows of their own and a bias of -1 (never selected)
    full = E // 3
    n_rows = full + E % 3
    grp = torch.where(perm < 3 * full, perm // 3, full + perm - 3 * full)
    rows = (0.02 * W.normal(W.stream_key(seed, TIE_TAG, E, d, 3), 0, n_rows * d)).to(torch.float32)
    gb = -0.01 + 0.02 * W.uniform01(W.stream_key(seed, TIE_TAG, E, d, 4), 0, n_rows)
    gb[full:] = -1.0
    return rows.view(n_rows, d)[grp].contiguous(), gb[grp].to(torch.float32).contiguous()


def tie_tokens(T: int, d: int, seed: int = 0) -> torch.Tensor:
    return W.normal(W.stream_key(seed, TIE_TAG, T, d, 5), 0, T * d).view(T, d).to(torch.float32)


def oracle_route(x, wr, bias, k):
    idx, w, _, _, sel = O.route(x, wr, bias, k, 2.5, want_scores=True)
    return idx, w, sel


def assert_ties_present(sel, idx, k):
    """The constructed inputs really tie at the k-th slot for every token: some
    expert outside the oracle's top-k has the k-th selection value."""
    for t in range(idx.shape[0]):
        kth = sel[t, idx[t, k - 1]]
        outside = np.setdiff1d(np.arange(sel.shape[1]), idx[t])
        assert (sel[t, outside] == kth).any(), f"token {t}: no exact tie at slot {k}"


ROUTE_CASES = [  # (kind, E, k, T): T <= 8 takes the router GEMV, larger T the tiled router
    ("zero", 8, 2, 5), ("dup", 8, 2, 7), ("zero", 64, 8, 3), ("dup", 64, 8, 8),
    ("zero", 256, 8, 1), ("dup", 256, 8, 4), ("zero", 256, 8, 40), ("dup", 256, 8, 72),
    ("zero", 512, 8, 6), ("dup", 512, 8, 33), ("zero", 1024, 32, 8), ("dup", 1024, 32, 8),
    ("zero", 1024, 32, 20), ("dup", 1024, 32, 45), ("dup", 24, 5, 13), ("zero", 24, 5, 2),
]


@pytest.mark.parametrize("kind,E,k,T", ROUTE_CASES)
def test_route_exact_ties(kind, E, k, T):
    d = 256
    wr, bias = tie_router(E, d, k, kind)
    x = tie_tokens(T, d)
    o_idx, o_w, o_sel = oracle_route(x, wr, bias, k)
    assert_ties_present(o_sel, o_idx, k)
    cfg = M.config(d, 128, E, k, 1, 4)
    ws = M.workspace(cfg, T)
    idx = torch.full((T, k), -1, dtype=torch.int32, device="cuda")
    w = torch.zeros(T, k, device="cuda")
    M.moe_route(cfg, x.cuda(), wr.cuda(), bias.cuda(), idx, w, ws)
    assert M.moe_poll_status(ws) == M.MOE_OK
    np.testing.assert_array_equal(idx.cpu().numpy(), o_idx)
    np.testing.assert_allclose(w.cpu().numpy(), o_w, rtol=2e-6, atol=1e-7)
    if T <= 8:  # the allocation-free router on the same inputs
        idx2 = torch.full((T, k), -1, dtype=torch.int32, device="cuda")
        w2 = torch.zeros(T, k, device="cuda")
        M.moe_route_static(cfg, x.cuda(), wr.cuda(), bias.cuda(), idx2, w2)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(idx2.cpu().numpy(), o_idx)
        np.testing.assert_allclose(w2.cpu().numpy(), o_w, rtol=2e-6, atol=1e-7)


LAYER_CASES = [  # (kind, E, k, T, path)
    ("zero", 8, 2, 1, "auto"), ("dup", 8, 2, 6, "auto"), ("dup", 256, 8, 1, "auto"), ("zero", 256, 8, 8, "auto"),
    ("dup", 512, 8, 1, "auto"), ("zero", 512, 8, 5, "auto"), ("dup", 1024, 32, 1, "auto"),
    ("dup", 1024, 32, 8, "auto"), ("dup", 512, 8, 32, "auto"), ("dup", 1024, 32, 32, "auto"),
    ("zero", 1024, 32, 12, "multi"), ("dup", 512, 8, 6, "multi"), ("dup", 256, 8, 24, "multi"),
    ("dup", 8, 2, 6, "decode"), ("zero", 256, 8, 8, "decode"), ("zero", 512, 8, 5, "decode"),
    ("dup", 1024, 32, 8, "decode"),
]


@pytest.mark.parametrize("kind,E,k,T,path", LAYER_CASES)
def test_layer_exact_ties_and_wide_pools(kind, E, k, T, path):
    """The whole layer on tying router inputs: routing exact against the
    oracle (no allowance) and the output within the layer tolerance.  E = 512
    and 1024 run the decode kernel's shared-memory top-k (T <= 8), the tiled
    router's top-k with the separate bucketing kernel and the tensor-core path
    (AUTO from 3 tokens on), and the dp4a multi-kernel path."""
    wl = W.workload(0).replace(name=f"ties_{kind}_E{E}", d=256, f=128, n_experts=E, top_k=k, T=T)
    wr, bias = tie_router(E, wl.d, k, kind)
    L = W.layer(wl, 0, 0)
    L = W.Layer(wl, 0, 0, L.scales, wr, bias)
    dl = W.device_layer(wl, 0, 0, host=L)
    x = tie_tokens(T, wl.d, seed=1)
    cfg = M.config(wl.d, wl.f, E, k, 1, 4)
    ws = M.workspace(cfg, T)
    out = torch.empty(T, wl.d, device="cuda")
    idx = torch.full((T, k), -1, dtype=torch.int32, device="cuda")
    w = torch.zeros(T, k, device="cuda")
    opts = M.MoeLayerOpts()
    opts.path = {"auto": M.MOE_PATH_AUTO, "multi": M.MOE_PATH_MULTI, "decode": M.MOE_PATH_DECODE}[path]
    M.moe_layer(cfg, M.make_pool(dl.pool_w, dl.pool_s), dl.w_router, dl.bias, x.cuda(), out, ws,
                topk_idx_out=idx, topk_w_out=w, opts=opts)
    assert M.moe_poll_status(ws) == M.MOE_OK
    expect = {"multi": M.MOE_PATH_MULTI, "decode": M.MOE_PATH_DECODE}.get(
        path, M.MOE_PATH_DECODE if T <= 2 else M.MOE_PATH_TC)
    assert opts.path_ran == expect
    r = O.workload_layer(wl, 0, 0, x, L=L)
    _, _, o_sel = oracle_route(x, wr, bias, k)
    assert_ties_present(o_sel, r["idx"], k)
    np.testing.assert_array_equal(idx.cpu().numpy(), r["idx"])
    np.testing.assert_allclose(w.cpu().numpy(), r["w"], rtol=2e-6, atol=1e-7)
    assert rel_l2(out.cpu().numpy(), r["out"]) <= OUT_REL_L2
