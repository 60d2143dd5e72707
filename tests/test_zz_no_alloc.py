"""moe_route_static: the router for callers that cannot allocate device memory.

Some callers of this library cannot hand it a workspace -- a host framework
that owns all device memory and forbids allocations after start-up, a serving
loop that must not pay cudaMalloc's implicit synchronisation, a plugin with no
way to ask for scratch space.  moe_route_static keeps its scratch in a fixed
array inside libmoe.so instead.  This test checks, through the C ABI, that two
calls in a row (which share that array) give the same routing as moe_route
with a caller-provided workspace, and that requests beyond its limit are
refused.  It sits in a file of its own, collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import expert_ffn_router_b200 as M
import oracle as O
import workloads as W
from parity_utils import routing_mismatches

FAKE = 1 << 20


def cfg_of(wl):
    return M.config(wl.d, wl.f, wl.n_experts, wl.top_k, wl.has_shared, wl.wbits, wl.routed_scale)


def test_static_router_rejects_requests_beyond_its_limit():
    wl = W.workload(1)
    c = cfg_of(wl)
    st = M.lib.moe_route_static(ctypes.byref(c), FAKE, 1, 9, FAKE, FAKE, FAKE, FAKE, None)
    assert st == M.MOE_EINVAL and b"limit" in M.lib.moe_last_error()
    assert M.lib.moe_route_static(ctypes.byref(c), FAKE, 1, 0, FAKE, FAKE, FAKE, FAKE, None) == M.MOE_OK


WIDE = W.workload(0).replace(name="tiny_E1024_k32", n_experts=1024, top_k=32, T=8)


@pytest.mark.gpu
@pytest.mark.parametrize("which,T", [(0, 5), (1, 1), (1, 8), ("wide", 8)])
def test_static_router_matches_workspace_router(which, T):
    """The E = 1024, k = 32 case is the largest the static limits allow: the
    router's logits fill the array's largest region, and the top-k uses all
    32 lanes of its warp; it is also checked against the CPU oracle."""
    wl = WIDE if which == "wide" else W.workload(which)
    cfg = cfg_of(wl)
    L = W.layer(wl, 0, 0)
    wr, bias = L.w_router.cuda(), L.bias.cuda()
    ws = M.workspace(cfg, T)
    for call in range(2):  # two calls in a row share the static scratch
        x = W.tokens(wl, 0, 11 + call, T).cuda()
        ref_idx = torch.empty(T, wl.top_k, dtype=torch.int32, device="cuda")
        ref_w = torch.empty(T, wl.top_k, device="cuda")
        M.moe_route(cfg, x, wr, bias, ref_idx, ref_w, ws)
        idx = torch.full((T, wl.top_k), -1, dtype=torch.int32, device="cuda")
        w = torch.full((T, wl.top_k), -1.0, device="cuda")
        M.moe_route_static(cfg, x, wr, bias, idx, w)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx.cpu().numpy())
        np.testing.assert_allclose(w.cpu().numpy(), ref_w.cpu().numpy(), rtol=2e-6, atol=1e-7)
        if which == "wide":
            o_idx, _, _, _, o_sel = O.route(x.float(), L.w_router, L.bias, wl.top_k, wl.routed_scale,
                                            want_scores=True)
            _, bad = routing_mismatches(idx.cpu().numpy(), o_idx, o_sel)
            assert bad == []
