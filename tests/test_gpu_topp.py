"""TOPK/TOPP truncation of the router (moe_config.topp) against the oracle.

Every router implementation and every layer path runs with truncation on:
the one-warp small router (T <= 8), the tiled router with its register top-k
and bucketing (E <= 256) or its shared-memory top-k and separate bucketing
(E > 256), the allocation-free router, the decode kernel (register and
shared-memory top-k, one-token row-range path at the GLM-5.2 expert shape,
several-token path), the dp4a multi-kernel path and the tensor-core path.
Routing must match the oracle's exactly (dropped slots -1, kept prefix and
weights), except on tokens where the float32 decision sits within 1e-5 of
its threshold or the selection within 1e-6 of a tie (counted; the oracle
takes the decision on its own scores); layer outputs within 2e-3 relative L2.
"""
import numpy as np
import pytest
import torch

import expert_ffn_router_b200 as M
import oracle as O
import workloads as W
from parity_utils import NEAR_TIE_REL, OUT_REL_L2, rel_l2

pytestmark = pytest.mark.gpu

NEAR_THRESHOLD_REL = 1e-5


def near_threshold(s_slots, p):
    """True if some slot's float32 prefix sum lies within NEAR_THRESHOLD_REL of
    the truncation threshold (the GPU's own scores could take the decision the
    other way)."""
    tot = np.float32(0.0)
    before = []
    for v in s_slots:
        before.append(tot)
        tot = np.float32(tot + np.float32(v))
    thr = np.float32(np.float32(p) * tot)
    return any(abs(float(b) - float(thr)) <= NEAR_THRESHOLD_REL * float(thr) for b in before[1:])


def compare_routing(g_idx, g_w, x, wr, bias, k, p, scale=2.5):
    """Returns the tokens allowed to differ; asserts everything else."""
    o_idx, o_w = O.route(x, wr, bias, k, scale, topp=p)
    full, _, _, s, sel = O.route(x, wr, bias, k, scale, want_scores=True)
    allowed = []
    for t in range(o_idx.shape[0]):
        g, o = g_idx[t], o_idx[t]
        if np.array_equal(g, o):
            kept = o >= 0
            np.testing.assert_allclose(g_w[t][kept], o_w[t][kept], rtol=2e-6, atol=1e-7)
            assert (g_w[t][~kept] == 0).all()
            continue
        m, gm = int((o >= 0).sum()), int((g >= 0).sum())
        tie = m == gm and all(abs(sel[t, g[j]] - sel[t, o[j]]) <= NEAR_TIE_REL * abs(sel[t, o[j]]) for j in range(m))
        assert near_threshold(s[t, full[t]], p) or tie, (t, g, o)
        allowed.append(t)
    return allowed


ROUTE_CASES = {  # name: (E, k, d, T, entry)
    "small_T5": (40, 6, 1056, 5, "route"),
    "tiled_T37_E64": (64, 8, 1024, 37, "route"),
    "tiled_T32_E512": (512, 8, 512, 32, "route"),
    "static_T8_E64": (64, 8, 1024, 8, "static"),
}


@pytest.mark.parametrize("p", [0.5, 0.8])
@pytest.mark.parametrize("name", list(ROUTE_CASES))
def test_route_truncation(name, p):
    E, k, d, T, entry = ROUTE_CASES[name]
    wl = W.workload(0).replace(name=f"topp_{name}", d=d, f=128, n_experts=E, top_k=k, T=T)
    L = W.layer(wl, 0, 0)
    x = W.tokens(wl, 0, 1).float()
    cfg = M.config(d, 128, E, k, 1, 4, 2.5, topp=p)
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, device="cuda")
    if entry == "static":
        M.moe_route_static(cfg, x.cuda(), L.w_router.cuda(), L.bias.cuda(), idx, w)
    else:
        ws = M.workspace(cfg, T)
        M.moe_route(cfg, x.cuda(), L.w_router.cuda(), L.bias.cuda(), idx, w, ws)
        assert M.moe_poll_status(ws) == M.MOE_OK
    torch.cuda.synchronize()
    g_idx, g_w = idx.cpu().numpy(), w.cpu().numpy()
    allowed = compare_routing(g_idx, g_w, x, L.w_router, L.bias, k, p)
    assert len(allowed) <= max(1, T // 10), allowed
    assert (g_idx == -1).any()  # the threshold does truncate on these inputs


LAYER_CASES = {  # name: (workload, path)
    "glm_T1_rowrange": (W.workload(1).replace(name="glm_e16_topp", n_experts=16, top_k=8, T=1), M.MOE_PATH_AUTO),
    "small_T1_decode": (W.workload(0).replace(name="tp1", d=2048, f=1024, n_experts=24, top_k=6, T=1), M.MOE_PATH_AUTO),
    "small_T5_decode": (W.workload(0).replace(name="tp5", d=1056, f=352, n_experts=40, top_k=6, T=5), M.MOE_PATH_DECODE),
    "small_T5_E512_decode": (W.workload(0).replace(name="tp5e", d=256, f=128, n_experts=512, top_k=8, T=5),
                             M.MOE_PATH_DECODE),
    "small_T5_multi": (W.workload(0).replace(name="tp5", d=1056, f=352, n_experts=40, top_k=6, T=5), M.MOE_PATH_MULTI),
    "small_T37_tc": (W.workload(0).replace(name="tp37", d=1056, f=352, n_experts=40, top_k=6, T=37), M.MOE_PATH_TC),
    "small_T37_multi": (W.workload(0).replace(name="tp37", d=1056, f=352, n_experts=40, top_k=6, T=37),
                        M.MOE_PATH_MULTI),
}


@pytest.mark.parametrize("name", list(LAYER_CASES))
def test_layer_truncation(name):
    base, path = LAYER_CASES[name]
    p = 0.7
    wl = base.replace(topp=p)
    L = W.layer(wl, 0, 0)
    dl = W.device_layer(wl, 0, 0, host=L)
    cfg = M.config(wl.d, wl.f, wl.n_experts, wl.top_k, wl.has_shared, wl.wbits, wl.routed_scale, topp=p)
    pool = M.make_pool(dl.pool_w, dl.pool_s)
    ws = M.workspace(cfg, wl.T)
    n_drop = 0
    for s_ in range(3 if wl.T == 1 else 1):
        x = W.tokens(wl, 0, s_)
        out = torch.full((wl.T, wl.d), float("nan"), device="cuda")
        idx = torch.empty(wl.T, wl.top_k, dtype=torch.int32, device="cuda")
        w = torch.empty(wl.T, wl.top_k, device="cuda")
        o = M.MoeLayerOpts()
        o.path = path
        M.moe_layer(cfg, pool, dl.w_router, dl.bias, x.cuda(), out, ws, topk_idx_out=idx, topk_w_out=w, opts=o)
        torch.cuda.synchronize()
        assert M.moe_poll_status(ws) == M.MOE_OK
        g_idx = idx.cpu().numpy()
        n_drop += int((g_idx == -1).sum())
        allowed = compare_routing(g_idx, w.cpu().numpy(), x.float(), L.w_router, L.bias, wl.top_k, p)
        r = O.workload_layer(wl, 0, 0, x.float(), L=L)
        keep = [t for t in range(wl.T) if t not in allowed]
        assert rel_l2(out.cpu().numpy()[keep], r["out"][keep]) <= OUT_REL_L2
    assert n_drop > 0
