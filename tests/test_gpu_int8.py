"""int8 expert weights (one two's-complement code per byte, per-row fp32
scales) at the GLM-5.2 expert shape, d = 6144, f = 2048, on a 32-expert pool
with the shared expert: every path against the CPU oracle.

A row of 6144 int8 codes is 384 16-byte chunks, 12 per lane of a warp (the
multi-kernel path's widest row); the tensor-core path takes them in 64-column
chunks.  One gate/up unit of the single-launch decode kernel (8 gate and 8 up
rows) is 96 KB here, so its ring keeps 2 slots instead of 4, one token runs by
whole units rather than by output-row ranges, and from 4 tokens on (whose
inputs and h rows take the room of the second slot) the kernel declines the
shape; AUTO takes the tensor-core path there anyway.
"""
import numpy as np
import pytest
import torch

import expert_ffn_router_b200 as M
import workloads as W
from test_gpu_parity import compare_layer, run_layer_gpu, x_host
from test_gpu_tc import run_layer_tc

pytestmark = pytest.mark.gpu

WL = W.workload(1).replace(name="glm_int8_e32", n_experts=32, wbits=8)


@pytest.fixture(scope="module")
def layer():
    L = W.layer(WL, 0, 0)
    return L, W.device_layer(WL, 0, 0, host=L)


def cfg():
    return M.config(WL.d, WL.f, WL.n_experts, WL.top_k, WL.has_shared, WL.wbits, WL.routed_scale)


def test_int8_one_token(layer):
    L, dl = layer
    ws = M.workspace(cfg(), 8)
    pool = M.make_pool(dl.pool_w, dl.pool_s)
    for s in range(4):
        x = x_host(WL, s, 1)
        out = torch.empty(1, WL.d, device="cuda")
        idx = torch.empty(1, WL.top_k, dtype=torch.int32, device="cuda")
        o = M.MoeLayerOpts()
        M.moe_layer(cfg(), pool, dl.w_router, dl.bias, x.cuda(), out, ws, topk_idx_out=idx, opts=o)
        assert M.moe_poll_status(ws) == M.MOE_OK
        assert o.path_ran == M.MOE_PATH_DECODE
        compare_layer(WL, L, x, out, idx.cpu().numpy())
        out_m, g_m, _ = run_layer_gpu(WL, dl, x, path="multi", ws=ws)
        compare_layer(WL, L, x, out_m, g_m)


@pytest.mark.parametrize("path,T", [("decode", 2), ("multi", 4), ("multi", 9)])
def test_int8_few_tokens(layer, path, T):
    L, dl = layer
    x = x_host(WL, 5, T)
    out, g_idx, _ = run_layer_gpu(WL, dl, x, path=path)
    compare_layer(WL, L, x, out, g_idx)


def test_int8_decode_declines_eight_tokens(layer):
    _, dl = layer
    with pytest.raises(M.MoeError, match="decode path"):
        run_layer_gpu(WL, dl, x_host(WL, 5, 8), path="decode")


@pytest.mark.parametrize("T", [16, 96])
def test_int8_tensor_core(layer, T):
    L, dl = layer
    x = x_host(WL, 7, T)
    out, g_idx, _ = run_layer_tc(WL, dl, x)
    tokens = list(range(T)) if T <= 16 else list(range(0, T, 7))
    compare_layer(WL, L, x, out, g_idx, tokens=tokens)
    # AUTO takes the tensor-core path here, bit for bit the same
    out2, g2, _ = run_layer_gpu(WL, dl, x)
    np.testing.assert_array_equal(g2, g_idx)
    assert torch.equal(out2, out)
