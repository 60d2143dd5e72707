"""The decode kernel's bounded waits: a wait that runs out ends the call with
MOE_ETIMEOUT in the workspace's status word instead of hanging.

Nothing faults: the test asks the kernel (moe_layer_opts.test_skip_h) to leave
one task's h values unwritten, so every wait on them -- the CTA that polls the
task's h values to requantise them, and every CTA polling for the codes it
publishes -- runs out after the given limit (wait_limit_us).  The call
returns, moe_poll_status reports MOE_ETIMEOUT with the site code of one of
those polls, and after moe_workspace_init the same workspace gives correct
results again.  The hook exists on the one-token row-range path, i.e. the
GLM-5.2 expert shape (d = 6144, f = 2048), here with a 16-expert pool.
"""
import numpy as np
import pytest
import torch

import expert_ffn_router_b200 as M
import oracle as O
import workloads as W
from parity_utils import OUT_REL_L2, rel_l2

pytestmark = pytest.mark.gpu

WL = W.workload(0).replace(name="glm_e16", d=6144, f=2048, n_experts=16, top_k=4, T=1, x_dtype="bf16")


def run(cfg, pool, dl, x, ws, opts):
    out = torch.empty(1, WL.d, device="cuda")
    idx = torch.empty(1, WL.top_k, dtype=torch.int32, device="cuda")
    M.moe_layer(cfg, pool, dl.w_router, dl.bias, x, out, ws, topk_idx_out=idx, opts=opts)
    return out, idx


@pytest.mark.parametrize("skip_task", [0, 2])
def test_wait_runs_out_and_reports(skip_task):
    L = W.layer(WL, 0, 0)
    dl = W.device_layer(WL, 0, 0, host=L)
    cfg = M.config(WL.d, WL.f, WL.n_experts, WL.top_k, WL.has_shared, WL.wbits, WL.routed_scale)
    pool = M.make_pool(dl.pool_w, dl.pool_s)
    ws = M.workspace(cfg, 1)
    x = W.tokens(WL, 0, 3).cuda()
    o = M.MoeLayerOpts()
    o.wait_limit_us = 1000
    o.test_skip_h = 1 + skip_task
    run(cfg, pool, dl, x, ws, o)
    torch.cuda.synchronize()
    assert o.path_ran == M.MOE_PATH_DECODE
    import ctypes
    info = ctypes.c_int32(0)
    st = M.lib.moe_poll_status(ws.data_ptr(), ctypes.byref(info), torch.cuda.current_stream().cuda_stream)
    # whichever wait on the missing values runs out first reports: the
    # requantising CTA's poll of the h values (410) or another CTA's poll of
    # the codes and scale it publishes (420)
    assert st == M.MOE_ETIMEOUT and info.value in (410, 420), (st, info.value)
    # the context is usable and the workspace recovers after initialisation
    M.moe_workspace_init(ws)
    out, idx = run(cfg, pool, dl, x, ws, M.MoeLayerOpts())
    assert M.moe_poll_status(ws) == M.MOE_OK
    r = O.workload_layer(WL, 0, 0, W.tokens(WL, 0, 3).float(), L=L)
    np.testing.assert_array_equal(idx.cpu().numpy(), r["idx"])
    assert rel_l2(out.cpu().numpy(), r["out"]) <= OUT_REL_L2
