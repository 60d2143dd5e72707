"""moe_layer with x and out in pinned host memory (moe_layer_opts.io_host).

The call copies x from mapped host memory into the workspace with a small
kernel and the kernels write out straight into host memory; the results must
be bit-identical to the same call on device buffers, on the decode kernel
(one token, the GLM-5.2 expert shape), the tensor-core path and the dp4a path,
in plain and accumulate mode.  Host argument errors are checked too.
"""
import numpy as np
import pytest
import torch

import expert_ffn_router_b200 as M
import workloads as W

pytestmark = pytest.mark.gpu

CASES = {
    "decode_glm_e16": (W.workload(1).replace(name="glm_e16", n_experts=16, top_k=4), M.MOE_PATH_AUTO),
    "tc_small_T16": (W.workload(0).replace(name="tc16", d=1024, f=512, n_experts=24, top_k=4, T=16), M.MOE_PATH_TC),
    "multi_small_T5": (W.workload(0).replace(name="multi5", d=1056, f=352, n_experts=40, top_k=6, T=5),
                       M.MOE_PATH_MULTI),
}


def setup(wl):
    dl = W.device_layer(wl, 0, 0)
    cfg = M.config(wl.d, wl.f, wl.n_experts, wl.top_k, wl.has_shared, wl.wbits, wl.routed_scale)
    return dl, cfg, M.make_pool(dl.pool_w, dl.pool_s), M.workspace(cfg, wl.T)


@pytest.mark.parametrize("name", list(CASES))
def test_host_io_matches_device_io(name):
    wl, path = CASES[name]
    dl, cfg, pool, ws = setup(wl)
    x = W.tokens(wl, 0, 2)
    xd = x.cuda()
    xh = x.pin_memory()
    ref = torch.empty(wl.T, wl.d, device="cuda")
    o = M.MoeLayerOpts()
    o.path = path
    M.moe_layer(cfg, pool, dl.w_router, dl.bias, xd, ref, ws, opts=o)
    for io in (M.MOE_IO_X_HOST, M.MOE_IO_OUT_HOST, M.MOE_IO_X_HOST | M.MOE_IO_OUT_HOST):
        xin = xh if io & M.MOE_IO_X_HOST else xd
        out = torch.full((wl.T, wl.d), float("nan")).pin_memory() if io & M.MOE_IO_OUT_HOST else \
            torch.empty(wl.T, wl.d, device="cuda")
        o = M.MoeLayerOpts()
        o.path = path
        o.io_host = io
        M.moe_layer(cfg, pool, dl.w_router, dl.bias, xin, out, ws, opts=o)
        torch.cuda.synchronize()
        assert M.moe_poll_status(ws) == M.MOE_OK
        assert o.path_ran == (M.MOE_PATH_DECODE if path == M.MOE_PATH_AUTO else path)
        assert torch.equal(out.cpu(), ref.cpu()), io
    # accumulate into host memory: base + the layer
    base = torch.randn(wl.T, wl.d)
    acc = base.clone().pin_memory()
    o = M.MoeLayerOpts()
    o.path = path
    o.io_host = M.MOE_IO_X_HOST | M.MOE_IO_OUT_HOST
    M.moe_layer(cfg, pool, dl.w_router, dl.bias, xh, acc, ws, accumulate=True, opts=o)
    torch.cuda.synchronize()
    np.testing.assert_allclose(acc.numpy(), (base + ref.cpu()).numpy(), rtol=1e-6, atol=1e-5)


def test_host_io_rejects_device_pointers_and_unknown_bits():
    wl, _ = CASES["multi_small_T5"]
    dl, cfg, pool, ws = setup(wl)
    x = W.tokens(wl, 0, 0).cuda()
    out = torch.empty(wl.T, wl.d, device="cuda")
    import ctypes
    for io in (M.MOE_IO_X_HOST, M.MOE_IO_OUT_HOST, 4):
        o = M.MoeLayerOpts()
        o.io_host = io
        st = M.lib.moe_layer_ex(ctypes.byref(cfg), ctypes.byref(pool), dl.w_router.data_ptr(), dl.bias.data_ptr(),
                                x.data_ptr(), M.MOE_F32, wl.T, out.data_ptr(), 0, None, None, ws.data_ptr(),
                                ws.numel(), torch.cuda.current_stream().cuda_stream, ctypes.byref(o))
        assert st == M.MOE_EINVAL, (io, st)
