"""The tensor-core (tcgen05 int8 grouped GEMM) expert path against the CPU
oracle, through the C ABI.

Forced with moe_config.tc_min_tokens = 1 (or the layer's MOE_PATH_TC).  Cases
span: padded token counts of 8 and 16 and a multiple of 16, tasks split at 64
tokens (130, 160, 300 tokens of one expert), ragged K (d = 1056: the last
128-column chunk is partly outside the row; f = 320 with int2: 256-column
chunks; int8 rows: 64-column chunks), ragged rows (f = 352: the last 128-row
tile is partly another matrix's rows), int8, int4 and int2 weights, routed and
shared experts, and the full d = 6144, f = 2048 shapes.  Integer accumulators
must be bit-exact.
"""
import numpy as np
import pytest
import torch

import expert_ffn_router_b200 as M
import oracle as O
import workloads as W
from parity_utils import HQ_MAX_FRAC, OUT_REL_L2, hq_close, rel_l2
from test_gpu_parity import SMALL, compare_layer, x_host, to_dev, assert_ok

pytestmark = pytest.mark.gpu


def cfg_tc(wl, thr=1):
    return M.config(wl.d, wl.f, wl.n_experts, wl.top_k, wl.has_shared, wl.wbits, wl.routed_scale, thr)


TC_EXPERT_CASES = [("tiny", 4, 1), ("tiny", 32, -1), ("ragged_int4", 9, 1), ("ragged_int4", 130, -1),
                   ("ragged_int2", 11, 2), ("ragged_int2", 40, -1), ("full_int4", 1, 7), ("full_int4", 160, -1),
                   ("full_int4", 300, 3), ("full_int2", 24, 5), ("ragged_int8", 9, 1), ("ragged_int8", 40, -1)]


def single_expert_pool(wl, e):
    blob = W.expert_blob(wl, 0, 0, e)
    sc = W.expert_scales(wl, 0, 0, e)
    pool_w = torch.zeros(wl.pool_bytes, dtype=torch.uint8, device="cuda")
    pool_w[e * wl.blob_bytes:(e + 1) * wl.blob_bytes] = blob.cuda()
    pool_s = torch.zeros(wl.n_blobs, wl.scale_rows, dtype=torch.float32, device="cuda")
    pool_s[e] = sc.cuda()
    return blob, sc, M.make_pool(pool_w, pool_s)


@pytest.mark.parametrize("name,T,expert", TC_EXPERT_CASES)
def test_tc_expert_stages(name, T, expert):
    if name.startswith("full"):
        wl = W.workload(1 if name == "full_int4" else 4)
    else:
        wl = SMALL[name]
    cfg = cfg_tc(wl)
    e = wl.n_experts if expert < 0 else expert
    blob, sc, pool = single_expert_pool(wl, e)
    x = W.tokens(wl, 0, 2, T).float()
    xq_o, sx_o = O.quantize(x)
    r = O.expert(wl.d, wl.f, wl.wbits, blob, sc, xq_o, sx_o)
    ws = M.workspace(cfg, T)
    y = torch.empty(T, wl.d, device="cuda")
    acc_gu = torch.empty(T, 2 * wl.f, dtype=torch.int32, device="cuda")
    hq = torch.empty(T, wl.f, dtype=torch.int8, device="cuda")
    sh = torch.empty(T, device="cuda")
    acc_d = torch.empty(T, wl.d, dtype=torch.int32, device="cuda")
    M.moe_expert_ffn(cfg, pool, expert, torch.from_numpy(xq_o).cuda(), torch.from_numpy(sx_o).cuda(), y, ws,
                     acc_gu, hq, sh, acc_d)
    assert_ok(ws)
    np.testing.assert_array_equal(acc_gu.cpu().numpy(), r["acc_gu"])
    mx, frac = hq_close(hq.cpu().numpy(), r["hq"])
    assert mx <= 1 and frac <= HQ_MAX_FRAC, (mx, frac)
    np.testing.assert_allclose(sh.cpu().numpy(), r["sh"], rtol=1e-6)
    assert rel_l2(y.cpu().numpy(), r["y"]) <= OUT_REL_L2
    # teacher-forced down on the oracle's codes: bit-exact accumulators
    y2 = torch.empty(T, wl.d, device="cuda")
    acc_d2 = torch.empty(T, wl.d, dtype=torch.int32, device="cuda")
    M.moe_expert_down(cfg, pool, expert, torch.from_numpy(r["hq"]).cuda(), torch.from_numpy(r["sh"]).cuda(), y2, ws,
                      acc_d2)
    assert_ok(ws)
    np.testing.assert_array_equal(acc_d2.cpu().numpy(), r["acc_d"])
    np.testing.assert_allclose(y2.cpu().numpy(), r["y"], rtol=1e-6, atol=1e-30)


def run_layer_tc(wl, dl, x, accumulate_into=None, ws=None, path=M.MOE_PATH_TC):
    cfg = cfg_tc(wl)
    T = x.shape[0]
    pool = M.make_pool(dl.pool_w, dl.pool_s)
    out = accumulate_into if accumulate_into is not None else torch.empty(T, wl.d, device="cuda")
    idx = torch.empty(T, wl.top_k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, wl.top_k, device="cuda")
    ws = M.workspace(cfg, T) if ws is None else ws
    opts = M.MoeLayerOpts()
    opts.path = path
    M.moe_layer(cfg, pool, dl.w_router, dl.bias, to_dev(x), out, ws, accumulate=accumulate_into is not None,
                topk_idx_out=idx, topk_w_out=w, opts=opts)
    assert_ok(ws)
    if path == M.MOE_PATH_TC:
        assert opts.path_ran == M.MOE_PATH_TC
        # router (T > 8: quantise, GEMM, top-k with the bucketing in its last CTA), gather, gate/up,
        # requantisation, down, combine
        assert opts.n_launches == (1 if T <= 8 else (3 if wl.n_experts <= 256 else 4)) + 5
    return out, idx.cpu().numpy(), w.cpu().numpy()


@pytest.mark.parametrize("name", list(SMALL))
def test_tc_layer_small(name):
    wl = SMALL[name]
    L = W.layer(wl, 0, 0)
    dl = W.device_layer(wl, 0, 0, host=L)
    x = x_host(wl)
    out, g_idx, _ = run_layer_tc(wl, dl, x)
    compare_layer(wl, L, x, out, g_idx)
    base = torch.randn(x.shape[0], wl.d, device="cuda")
    acc, _, _ = run_layer_tc(wl, dl, x, accumulate_into=base.clone())
    np.testing.assert_allclose(acc.cpu().numpy(), (base + out).cpu().numpy(), rtol=1e-6, atol=1e-5)


@pytest.mark.parametrize("T", [1, 16, 100])
def test_tc_layer_decode_shape(T):
    """The full d = 6144, 256-expert layer on the tensor-core path at
    decode-like token counts (one token per task up to a few)."""
    wl = W.workload(1)
    L = W.layer(wl, 0, 0)
    dl = W.device_layer(wl, 0, 0, host=L)
    x = x_host(wl, 7, T)
    out, g_idx, _ = run_layer_tc(wl, dl, x)
    tokens = list(range(0, T, max(1, T // 12)))
    err, _ = compare_layer(wl, L, x, out, g_idx, tokens)
    print(f"tensor-core layer T={T}: rel L2 {err:.3g}")


def test_tc_layer_prefill_sampled_matches_multi():
    """Prefill (T = 512, outlier channels): the tensor-core layer against the
    oracle on sampled tokens, and against the dp4a multi-kernel layer on
    every token (both compute the same integer dots; outputs differ only by
    the requantisation's half-point ulps)."""
    wl = W.workload(3)
    L = W.layer(wl, 0, 0)
    dl = W.device_layer(wl, 0, 0, host=L)
    x = x_host(wl)
    out, g_idx, _ = run_layer_tc(wl, dl, x)
    tokens = list(range(0, wl.T, 64)) + [wl.T - 1]
    err, _ = compare_layer(wl, L, x, out, g_idx, tokens)
    out_m, idx_m, _ = run_layer_tc(wl, dl, x, path=M.MOE_PATH_MULTI)
    np.testing.assert_array_equal(g_idx, idx_m)
    assert rel_l2(out.cpu().numpy(), out_m.cpu().numpy()) <= 1e-3
    print("prefill tensor-core sampled rel L2:", err)


def test_tc_layer_hot_experts_split_tasks():
    """Skewed routing at T = 512 (the int2 workload's Zipf-biased router, one
    layer): the most-loaded experts receive well over 64 tokens, so their
    assignments are cut into several tensor-core tasks and their weights are
    read once per task.  The tokens of the hottest expert on both sides of
    each task boundary, and its first and last, against the oracle; every
    token against the dp4a multi-kernel layer."""
    wl = W.workload(4).replace(name="skewed_int2_T512", T=512, n_layers=1)
    L = W.layer(wl, 0, 0)
    dl = W.device_layer(wl, 0, 0, host=L)
    x = x_host(wl, 3, wl.T)
    out, g_idx, _ = run_layer_tc(wl, dl, x)
    counts = np.bincount(g_idx[g_idx >= 0].ravel(), minlength=wl.n_experts)
    hot = int(counts.argmax())
    assert counts[hot] > 2 * 64, counts[hot]  # at least three tasks
    hot_tokens = np.nonzero((g_idx == hot).any(axis=1))[0]  # (token, slot) order = task order
    picks = {0, len(hot_tokens) - 1}
    for b in range(64, len(hot_tokens), 64):
        picks |= {b - 1, b}
    tokens = sorted({int(hot_tokens[i]) for i in picks})
    err, _ = compare_layer(wl, L, x, out, g_idx, tokens)
    out_m, idx_m, _ = run_layer_tc(wl, dl, x, path=M.MOE_PATH_MULTI)
    np.testing.assert_array_equal(g_idx, idx_m)
    assert rel_l2(out.cpu().numpy(), out_m.cpu().numpy()) <= 1e-3
    print(f"hottest expert {hot}: {counts[hot]} tokens, {len(tokens)} sampled, rel L2 {err:.3g}")


def test_tc_workspace_reuse_deterministic():
    """Calls of different T alternating the tensor-core and decode paths on one
    workspace: counters self-reset, results identical call to call."""
    wl = SMALL["ragged_int4"]
    L = W.layer(wl, 0, 0)
    dl = W.device_layer(wl, 0, 0, host=L)
    cfg = cfg_tc(wl, 16)
    ws = M.workspace(cfg, 160)
    pool = M.make_pool(dl.pool_w, dl.pool_s)
    outs = []
    for T in (160, 1, 37, 160, 37):
        x = to_dev(x_host(wl, T, T))
        out = torch.empty(T, wl.d, device="cuda")
        M.moe_layer(cfg, pool, dl.w_router, dl.bias, x, out, ws)
        outs.append(out)
    assert M.moe_poll_status(ws) == M.MOE_OK
    assert torch.equal(outs[0], outs[3]) and torch.equal(outs[2], outs[4])
    # a decode call after a tensor-core call sees the counters it expects
    d_out = torch.empty(1, wl.d, device="cuda")
    M.moe_layer(cfg, pool, dl.w_router, dl.bias, to_dev(x_host(wl, 1, 1)), d_out, ws)
    d_ref = torch.empty(1, wl.d, device="cuda")
    M.moe_layer(cfg, pool, dl.w_router, dl.bias, to_dev(x_host(wl, 1, 1)), d_ref, M.workspace(cfg, 160))
    torch.cuda.synchronize()
    assert torch.equal(outs[1], d_out) and torch.equal(d_out, d_ref)
    r_out, r_idx, _ = run_layer_tc(wl, dl, x_host(wl, 160, 160))
    assert torch.equal(outs[0], r_out)  # same result from a fresh workspace
    compare_layer(wl, L, x_host(wl, 160, 160), outs[0], r_idx, list(range(0, 160, 16)))
