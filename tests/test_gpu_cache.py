"""The HBM expert cache with host-memory overflow (moe_cache_init /
moe_cache_fetch, moe_pool.slot_of).

The layer's pool sits in pinned host memory; a cache of fewer slots than
experts serves a sequence of calls: route, copy the indices to the host,
fetch, run the layer on the cached pool.  Outputs must be bit-identical to
the same calls on the full pool in device memory -- on the decode kernel (the
one-token row-range path at the GLM-5.2 expert shape, the several-token
path), the dp4a path and the tensor-core path -- while experts are evicted
and fetched again; the hit/miss counts are checked against the distinct
experts of each call; a cache too small for one call is refused.
"""
import ctypes

import pytest
import torch

import expert_ffn_router_b200 as M
import workloads as W

pytestmark = pytest.mark.gpu

CASES = {  # name: (workload, tokens per call, path, slots)
    "glm_T1_rowrange": (W.workload(1).replace(name="glm_e24c", n_experts=24, top_k=8, T=1), 1, M.MOE_PATH_AUTO, 13),
    "small_T1": (W.workload(0).replace(name="c1", d=1056, f=352, n_experts=40, top_k=6), 1, M.MOE_PATH_AUTO, 10),
    "small_T5_decode": (W.workload(0).replace(name="c5", d=1056, f=352, n_experts=40, top_k=6), 5, M.MOE_PATH_DECODE,
                        33),
    "small_T5_multi": (W.workload(0).replace(name="c5", d=1056, f=352, n_experts=40, top_k=6), 5, M.MOE_PATH_MULTI,
                       33),
    "small_T8_tc": (W.workload(0).replace(name="c8", d=1024, f=512, n_experts=64, top_k=6), 8, M.MOE_PATH_TC, 52),
    "small_T1_topp": (W.workload(0).replace(name="c1", d=1056, f=352, n_experts=40, top_k=6, topp=0.6), 1,
                      M.MOE_PATH_AUTO, 8),
}


@pytest.mark.parametrize("name", list(CASES))
def test_cached_layer_matches_resident_pool(name):
    wl, T, path, n_slots = CASES[name]
    dl = W.device_layer(wl, 0, 0)
    cfg = M.config(wl.d, wl.f, wl.n_experts, wl.top_k, wl.has_shared, wl.wbits, wl.routed_scale, topp=wl.topp)
    full = M.make_pool(dl.pool_w, dl.pool_s)
    cache = M.ExpertCache(cfg, dl.pool_w.cpu().pin_memory(), dl.pool_s, n_slots)
    ws = M.workspace(cfg, T)
    ws2 = M.workspace(cfg, T)
    hits = misses = 0
    for call in range(12):
        x = W.tokens(wl, 0, call, T).cuda()
        idx = torch.empty(T, wl.top_k, dtype=torch.int32, device="cuda")
        w = torch.empty(T, wl.top_k, device="cuda")
        M.moe_route(cfg, x, dl.w_router, dl.bias, idx, w, ws)
        idx_h = idx.cpu()
        st = cache.fetch(idx_h)
        need = set(idx_h.reshape(-1).tolist()) - {-1}
        assert st.hits + st.misses == len(need)
        assert st.bytes == st.misses * cfg.blob_bytes
        hits, misses = hits + st.hits, misses + st.misses
        o = M.MoeLayerOpts()
        o.path = path
        out = torch.empty(T, wl.d, device="cuda")
        M.moe_layer(cfg, cache.pool, dl.w_router, dl.bias, x, out, ws, opts=o)
        o2 = M.MoeLayerOpts()
        o2.path = path
        ref = torch.empty(T, wl.d, device="cuda")
        M.moe_layer(cfg, full, dl.w_router, dl.bias, x, ref, ws2, opts=o2)
        torch.cuda.synchronize()
        assert M.moe_poll_status(ws) == M.MOE_OK and M.moe_poll_status(ws2) == M.MOE_OK
        assert o.path_ran == o2.path_ran
        assert torch.equal(out, ref), call
    # the cache was too small for every expert used: experts were evicted and fetched again
    assert misses > n_slots - wl.has_shared and hits > 0


def test_cache_refuses_a_call_it_cannot_hold():
    wl = W.workload(0).replace(name="c5", d=1056, f=352, n_experts=40, top_k=6)
    dl = W.device_layer(wl, 0, 0)
    cfg = M.config(wl.d, wl.f, wl.n_experts, wl.top_k, wl.has_shared, wl.wbits, wl.routed_scale)
    cache = M.ExpertCache(cfg, dl.pool_w.cpu().pin_memory(), dl.pool_s, 4)
    idx = torch.arange(6, dtype=torch.int32).view(1, 6)  # six experts, three free slots
    st = M.MoeCacheStats()
    rc = M.lib.moe_cache_fetch(ctypes.byref(cfg), ctypes.byref(cache.c), idx.data_ptr(), 1,
                               torch.cuda.current_stream().cuda_stream, ctypes.byref(st))
    assert rc == M.MOE_ENOSPACE
    assert cache.fetch(torch.tensor([[0, 1, 2, 0, 1, 2]], dtype=torch.int32)).misses == 3  # three distinct fit
