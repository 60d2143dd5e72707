"""CUDA path vs the CPU oracle on the same seeded inputs, through the C ABI.

Small shapes span several row blocks, a ragged lane tail (16-byte chunks per
row not a multiple of 32) and both router paths (GEMV for T <= 8, tiled for
larger T); full shapes are the decode, MTP-verify, prefill and skewed int2
workloads, checked on every token the oracle can afford (all of them for the
decode-sized ones, a sample for prefill and the 24-layer stack).
"""
import numpy as np
import pytest
import torch

import expert_ffn_router_b200 as M
import oracle as O
import workloads as W
from parity_utils import HQ_MAX_FRAC, OUT_REL_L2, hq_close, rel_l2, routing_mismatches

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny": W.workload(0),
    "ragged_int4": W.workload(0).replace(name="ragged_int4", d=1056, f=352, n_experts=40, top_k=6, T=37),
    "ragged_int4_T5": W.workload(0).replace(name="ragged_int4", d=1056, f=352, n_experts=40, top_k=6, T=5),
    "ragged_int2": W.workload(0).replace(name="ragged_int2", d=1088, f=320, n_experts=24, top_k=5, T=13, wbits=2),
    "k_eq_E": W.workload(0).replace(name="k_eq_E", d=256, f=128, n_experts=4, top_k=4, T=9),
    "no_shared": W.workload(0).replace(name="no_shared", d=512, f=256, n_experts=16, top_k=3, T=3,
                                       has_shared=0),
    "tiny_T1": W.workload(0).replace(name="tiny", T=1),
    "tiny_T8": W.workload(0).replace(name="tiny", T=8),
    "ragged_int2_T2": W.workload(0).replace(name="ragged_int2", d=1088, f=320, n_experts=24, top_k=5, T=2,
                                            wbits=2),
    "wide_k": W.workload(0).replace(name="wide_k", d=256, f=96, n_experts=64, top_k=32, T=7),
    "ragged_int8": W.workload(0).replace(name="ragged_int8", d=1056, f=352, n_experts=24, top_k=5, T=13, wbits=8),
    "ragged_int8_T2": W.workload(0).replace(name="ragged_int8", d=1056, f=352, n_experts=24, top_k=5, T=2,
                                            wbits=8),
}
PATHS = {"auto": M.MOE_PATH_AUTO, "multi": M.MOE_PATH_MULTI, "decode": M.MOE_PATH_DECODE}


def auto_path(T):
    """The path MOE_PATH_AUTO takes for T tokens with the default
    tc_min_tokens (3) on shapes that fit both kernels."""
    return M.MOE_PATH_DECODE if T <= 2 else M.MOE_PATH_TC

# One-token decode on small pools of d = 2048 (the decode kernel's runtime-loop
# rows): int4, int2 and int8 rows, no shared expert, E > 256 (its shared-memory
# top-k) and k = 32.
SINGLE = {
    "s1_int4": W.workload(0).replace(name="s1_int4", d=2048, f=1024, n_experts=16, top_k=4, T=1, x_dtype="bf16"),
    "s1_int2": W.workload(0).replace(name="s1_int2", d=2048, f=2048, n_experts=24, top_k=5, T=1, wbits=2,
                                     x_dtype="bf16"),
    "s1_no_shared": W.workload(0).replace(name="s1_no_shared", d=2048, f=1024, n_experts=12, top_k=3, T=1,
                                          has_shared=0),
    "s1_E512": W.workload(0).replace(name="s1_E512", d=2048, f=1024, n_experts=512, top_k=8, T=1),
    "s1_k32": W.workload(0).replace(name="s1_k32", d=2048, f=1024, n_experts=64, top_k=32, T=1),
    "s1_int8": W.workload(0).replace(name="s1_int8", d=2048, f=1024, n_experts=16, top_k=4, T=1, wbits=8,
                                     x_dtype="bf16"),
}


def cfg_of(wl):
    return M.config(wl.d, wl.f, wl.n_experts, wl.top_k, wl.has_shared, wl.wbits, wl.routed_scale)


def x_host(wl, token_set=0, T=None):
    return W.tokens(wl, 0, token_set, T)


def to_dev(t):
    return t.contiguous().cuda()


def assert_ok(ws):
    assert M.moe_poll_status(ws) == M.MOE_OK


@pytest.mark.parametrize("name", list(SMALL) + ["bf16_d6144"])
def test_quantize_bitexact(name):
    wl = SMALL.get(name) or W.workload(1)
    x = x_host(wl, 3, 64 if name == "bf16_d6144" else None)
    x[x.shape[0] // 2].zero_()  # an all-zero token
    q_o, s_o = O.quantize(x.float())
    xq = torch.empty(x.shape, dtype=torch.int8, device="cuda")
    sx = torch.empty(x.shape[0], dtype=torch.float32, device="cuda")
    M.moe_quantize(cfg_of(wl), to_dev(x), xq, sx)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(xq.cpu().numpy(), q_o)
    np.testing.assert_array_equal(sx.cpu().numpy(), s_o)


def check_route(wl, x, L, report):
    cfg = cfg_of(wl)
    T = x.shape[0]
    idx = torch.empty(T, wl.top_k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, wl.top_k, dtype=torch.float32, device="cuda")
    ws = M.workspace(cfg, T)
    M.moe_route(cfg, to_dev(x), to_dev(L.w_router), to_dev(L.bias), idx, w, ws)
    assert_ok(ws)
    o_idx, o_w, _, _, o_sel = O.route(x.float(), L.w_router, L.bias, wl.top_k, wl.routed_scale, want_scores=True)
    g_idx = idx.cpu().numpy()
    allowed, bad = routing_mismatches(g_idx, o_idx, o_sel)
    assert bad == [], f"routing differs beyond the near-tie rule on tokens {bad}"
    report.append((wl.name, T, len(allowed)))
    keep = [t for t in range(T) if t not in allowed]
    np.testing.assert_allclose(w.cpu().numpy()[keep], o_w[keep], rtol=2e-6, atol=1e-7)
    return g_idx


@pytest.mark.parametrize("name", list(SMALL))
def test_route_small(name):
    wl = SMALL[name]
    rep = []
    check_route(wl, x_host(wl), W.layer(wl, 0, 0), rep)


@pytest.mark.parametrize("T", [1, 4, 8, 64, 512])
def test_route_full_size(T):
    wl = W.workload(4 if T == 64 else 1)
    rep = []
    check_route(wl, x_host(wl, 1, T), W.layer(wl, 0, 0), rep)
    print("near-tie routing mismatches:", rep)


EXPERT_CASES = [("tiny", 4, 1), ("ragged_int4", 9, 1), ("ragged_int4", 3, -1), ("ragged_int2", 11, 2),
                ("full_int4", 1, 7), ("full_int4", 9, -1), ("full_int2", 3, 5), ("ragged_int8", 9, 1),
                ("ragged_int8", 3, -1)]


@pytest.mark.parametrize("name,T,expert", EXPERT_CASES)
def test_expert_stages(name, T, expert):
    if name.startswith("full"):
        wl = W.workload(1 if name == "full_int4" else 4)
    else:
        wl = SMALL[name]
    cfg = cfg_of(wl)
    e = wl.n_experts if expert < 0 else expert
    blob = W.expert_blob(wl, 0, 0, e)
    sc = W.expert_scales(wl, 0, 0, e)
    # a device pool holding only this expert's blob at its slot (others zero)
    pool_w = torch.zeros(wl.pool_bytes, dtype=torch.uint8, device="cuda")
    pool_w[e * wl.blob_bytes:(e + 1) * wl.blob_bytes] = blob.cuda()
    pool_s = torch.zeros(wl.n_blobs, wl.scale_rows, dtype=torch.float32, device="cuda")
    pool_s[e] = sc.cuda()
    pool = M.make_pool(pool_w, pool_s)
    x = x_host(wl, 2, T).float()
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
    # teacher-forced down on the oracle's codes: bit-exact accumulators
    y2 = torch.empty(T, wl.d, device="cuda")
    acc_d2 = torch.empty(T, wl.d, dtype=torch.int32, device="cuda")
    M.moe_expert_down(cfg, pool, expert, torch.from_numpy(r["hq"]).cuda(), torch.from_numpy(r["sh"]).cuda(), y2, ws,
                      acc_d2)
    assert_ok(ws)
    np.testing.assert_array_equal(acc_d2.cpu().numpy(), r["acc_d"])
    np.testing.assert_allclose(y2.cpu().numpy(), r["y"], rtol=1e-6, atol=1e-30)
    # the fused path's output against the oracle's
    assert rel_l2(y.cpu().numpy(), r["y"]) <= OUT_REL_L2


def run_layer_gpu(wl, dl, x, accumulate_into=None, path="auto", ws=None):
    cfg = cfg_of(wl)
    T = x.shape[0]
    pool = M.make_pool(dl.pool_w, dl.pool_s)
    out = accumulate_into if accumulate_into is not None else torch.empty(T, wl.d, device="cuda")
    idx = torch.empty(T, wl.top_k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, wl.top_k, device="cuda")
    ws = M.workspace(cfg, T) if ws is None else ws
    opts = M.MoeLayerOpts()
    opts.path = PATHS[path]
    M.moe_layer(cfg, pool, dl.w_router, dl.bias, to_dev(x), out, ws, accumulate=accumulate_into is not None,
                topk_idx_out=idx, topk_w_out=w, opts=opts)
    assert_ok(ws)
    if path == "auto":
        assert opts.path_ran == auto_path(T)
    if path == "decode":
        assert opts.n_launches == 1 and opts.path_ran == M.MOE_PATH_DECODE  # the single-launch kernel ran
    if path == "multi":
        assert opts.path_ran == M.MOE_PATH_MULTI
    return out, idx.cpu().numpy(), w.cpu().numpy()


def compare_layer(wl, L, x, out, g_idx, tokens=None):
    xf = x.float()
    if tokens is not None:
        xf = xf[tokens]
        out = out[tokens]
        g_idx = g_idx[tokens]
    r = O.workload_layer(wl, 0, 0, xf, L=L)
    _, _, _, _, o_sel = O.route(xf, L.w_router, L.bias, wl.top_k, wl.routed_scale, want_scores=True)
    allowed, bad = routing_mismatches(g_idx, r["idx"], o_sel)
    assert bad == [], bad
    keep = [t for t in range(xf.shape[0]) if t not in allowed]
    err = rel_l2(out.cpu().numpy()[keep], r["out"][keep])
    assert err <= OUT_REL_L2, err
    return err, allowed


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("name", list(SMALL))
def test_layer_small(name, path):
    wl = SMALL[name]
    if path == "decode" and wl.T > 8:
        pytest.skip("the decode kernel takes at most 8 tokens")
    L = W.layer(wl, 0, 0)
    dl = W.device_layer(wl, 0, 0, host=L)
    x = x_host(wl)
    out, g_idx, _ = run_layer_gpu(wl, dl, x, path=path)
    compare_layer(wl, L, x, out, g_idx)
    # accumulate mode adds the layer to what is there
    base = torch.randn(x.shape[0], wl.d, device="cuda")
    acc, _, _ = run_layer_gpu(wl, dl, x, accumulate_into=base.clone(), path=path)
    np.testing.assert_allclose(acc.cpu().numpy(), (base + out).cpu().numpy(), rtol=1e-6, atol=1e-5)


def test_layer_decode_full_size():
    """The decode workload as the bench runs it: T = 1 per call, 8 token sets,
    one workspace reused across calls; then T = 8 on the decode kernel and on
    AUTO's tensor-core path, and the multi-kernel path."""
    wl = W.workload(1)
    L = W.layer(wl, 0, 0)
    dl = W.device_layer(wl, 0, 0, host=L)
    ws = M.workspace(cfg_of(wl), 8)
    errs = []
    for s in range(8):
        x = x_host(wl, s)
        out, g_idx, _ = run_layer_gpu(wl, dl, x, ws=ws)
        err, allowed = compare_layer(wl, L, x, out, g_idx)
        errs.append(err)
    x = x_host(wl, 20, 8)
    out, g_idx, _ = run_layer_gpu(wl, dl, x, path="decode", ws=ws)
    errs.append(compare_layer(wl, L, x, out, g_idx)[0])
    out, g_idx, _ = run_layer_gpu(wl, dl, x, ws=ws)  # AUTO: the tensor-core path at 8 tokens
    errs.append(compare_layer(wl, L, x, out, g_idx)[0])
    out, g_idx, _ = run_layer_gpu(wl, dl, x_host(wl, 0), path="multi", ws=ws)
    errs.append(compare_layer(wl, L, x_host(wl, 0), out, g_idx)[0])
    print("decode rel L2 per call:", errs)


def test_layer_decode_repeats_bit_identical():
    """The single-token decode layer called 300 times on 6 tokens in turn,
    with an L2 flush before every other call: each token's output repeats bit
    for bit.  Its gate/up -> down hand-off has no fence (readers poll values
    preset to "not written"), so a stale or torn read would show here as a
    differing output (the outputs' agreement with the oracle is
    test_layer_decode_full_size's; each token's first output, the reference
    of the repeats, is also checked against the oracle here, so that a race
    on a first call cannot set a wrong reference)."""
    wl = W.workload(1)
    L = W.layer(wl, 0, 0)
    dl = W.device_layer(wl, 0, 0, host=L)
    cfg = cfg_of(wl)
    pool = M.make_pool(dl.pool_w, dl.pool_s)
    ws = M.workspace(cfg, 1)
    out = torch.empty(1, wl.d, device="cuda")
    idx = torch.empty(1, wl.top_k, dtype=torch.int32, device="cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    xs = [x_host(wl, s) for s in range(6)]
    toks = [to_dev(x) for x in xs]
    refs, ref_idx, bad = {}, {}, 0
    for it in range(300):
        i = it % 6
        if it % 2 == 0:
            flush.fill_(it & 0xFF)
        M.moe_layer(cfg, pool, dl.w_router, dl.bias, toks[i], out, ws, topk_idx_out=idx)
        o = out.clone()
        if i in refs:
            bad += int(not torch.equal(o, refs[i]))
        else:
            refs[i] = o
            ref_idx[i] = idx.cpu().numpy().copy()
    torch.cuda.synchronize()
    assert_ok(ws)
    assert bad == 0
    for i in range(6):
        compare_layer(wl, L, xs[i], refs[i], ref_idx[i])


def test_layer_decode_int2_full_size():
    wl = W.workload(4)
    L = W.layer(wl, 0, 0)
    dl = W.device_layer(wl, 0, 0, host=L)
    for T in (1, 3):
        x = x_host(wl, 5, T)
        out, g_idx, _ = run_layer_gpu(wl, dl, x)
        compare_layer(wl, L, x, out, g_idx)


def test_layer_prefill_sampled():
    wl = W.workload(3)
    L = W.layer(wl, 0, 0)
    dl = W.device_layer(wl, 0, 0, host=L)
    x = x_host(wl)
    out, g_idx, _ = run_layer_gpu(wl, dl, x)
    tokens = list(range(0, wl.T, 64)) + [wl.T - 1]
    err, _ = compare_layer(wl, L, x, out, g_idx, tokens)
    print("prefill sampled rel L2:", err)


def run_stack(wl, n_layers, token_subset):
    """GPU stack over every token; the oracle's own stack over a token subset."""
    T = wl.T
    x0 = x_host(wl)
    resid = torch.empty(T, wl.d, device="cuda")
    x_in = torch.empty(T, wl.d, device="cuda")
    M.moe_rmsnorm(to_dev(x0), x_in, 1e-6, x_copy=resid)
    idxs = []
    for l in range(n_layers):
        if l > 0:
            M.moe_rmsnorm(resid, x_in, 1e-6)
        dl = W.device_layer(wl, 0, l)
        _, g_idx, _ = run_layer_gpu(wl, dl, x_in, accumulate_into=resid)
        idxs.append(g_idx)
        del dl
    torch.cuda.synchronize()
    r = O.workload_stack(wl, 0, x0[token_subset], n_layers)
    return resid.cpu().numpy()[token_subset], idxs, r


@pytest.mark.parametrize("which,n_layers,tokens", [(2, 8, [0, 1, 2, 3]), (4, 24, [0, 21, 37, 63])])
def test_stacked_layers(which, n_layers, tokens):
    wl = W.workload(which)
    g_x, g_idxs, r = run_stack(wl, n_layers, tokens)
    diverged = set()
    for l in range(n_layers):
        L = W.layer(wl, 0, l)
        _, _, _, _, sel = O.route(r["x_in"][l], L.w_router, L.bias, wl.top_k, wl.routed_scale, want_scores=True)
        allowed, bad = routing_mismatches(g_idxs[l][tokens], r["idx"][l], sel)
        assert bad == [] or set(bad) <= diverged, (l, bad)
        diverged |= {tokens[i] for i in allowed + bad}
    keep = [i for i, t in enumerate(tokens) if t not in diverged]
    assert keep, "every sampled token hit a near-tie"
    err = rel_l2(g_x[keep], r["x"][keep])
    print(f"stack {wl.name}: final residual rel L2 {err:.3g}, near-tie tokens {sorted(diverged)}")
    assert err <= OUT_REL_L2


def test_workspace_reuse_and_status():
    """Back-to-back calls on one workspace stay correct (self-resetting counters)."""
    wl = SMALL["ragged_int4"]
    L = W.layer(wl, 0, 0)
    dl = W.device_layer(wl, 0, 0, host=L)
    cfg = cfg_of(wl)
    ws = M.workspace(cfg, wl.T)
    pool = M.make_pool(dl.pool_w, dl.pool_s)
    outs = []
    for T in (wl.T, 1, 5, wl.T, 5):  # alternates the multi-kernel and the single-launch paths
        x = to_dev(x_host(wl, T, T))
        out = torch.empty(T, wl.d, device="cuda")
        M.moe_layer(cfg, pool, dl.w_router, dl.bias, x, out, ws)
        outs.append(out)
    assert M.moe_poll_status(ws) == M.MOE_OK
    ref = torch.empty_like(outs[0])
    ws2 = M.workspace(cfg, wl.T)
    M.moe_layer(cfg, pool, dl.w_router, dl.bias, to_dev(x_host(wl, wl.T, wl.T)), ref, ws2)
    torch.cuda.synchronize()
    assert torch.equal(outs[0], ref) and torch.equal(outs[3], ref)  # deterministic
    assert torch.equal(outs[2], outs[4])


@pytest.mark.parametrize("name", list(SINGLE))
def test_layer_one_token_small_pools(name):
    """One token through the decode kernel on small pools (its runtime-loop
    rows; E up to 512, top-k up to 32): 6 tokens in turn on one workspace,
    each against the oracle; then the accumulate mode."""
    wl = SINGLE[name]
    L = W.layer(wl, 0, 0)
    dl = W.device_layer(wl, 0, 0, host=L)
    cfg = cfg_of(wl)
    pool = M.make_pool(dl.pool_w, dl.pool_s)
    ws = M.workspace(cfg, 1)
    for s_ in range(6):
        x = x_host(wl, s_)
        out = torch.empty(1, wl.d, device="cuda")
        idx = torch.empty(1, wl.top_k, dtype=torch.int32, device="cuda")
        o = M.MoeLayerOpts()
        M.moe_layer(cfg, pool, dl.w_router, dl.bias, to_dev(x), out, ws, topk_idx_out=idx, opts=o)
        assert_ok(ws)
        assert o.path_ran == M.MOE_PATH_DECODE
        compare_layer(wl, L, x, out, idx.cpu().numpy())
    base = torch.randn(1, wl.d, device="cuda")
    acc = base.clone()
    M.moe_layer(cfg, pool, dl.w_router, dl.bias, to_dev(x), acc, ws, accumulate=True)
    assert_ok(ws)
    np.testing.assert_allclose(acc.cpu().numpy(), (base + out).cpu().numpy(), rtol=1e-6, atol=1e-5)


@pytest.mark.parametrize("E", [8, 16, 24])
def test_layer_decode_few_experts_many_calls(E):
    """One token at the GLM-5.2 expert shape with pools of few experts: most
    CTAs own no router row and reach their first shared-expert unit right
    after quantising, while other CTAs still preset the call's h rows; the h
    values of that unit are stored only after the grid barrier, so none is
    erased by a late preset (which made the hand-off's poll run out).  60
    calls, every status OK, and each token's output against the oracle."""
    wl = W.workload(1).replace(name=f"glm_few_e{E}", n_experts=E, top_k=min(8, E))
    L = W.layer(wl, 0, 0)
    dl = W.device_layer(wl, 0, 0, host=L)
    cfg = cfg_of(wl)
    pool = M.make_pool(dl.pool_w, dl.pool_s)
    ws = M.workspace(cfg, 1)
    outs, idxs, xs = {}, {}, [x_host(wl, s) for s in range(3)]
    for it in range(60):
        out = torch.empty(1, wl.d, device="cuda")
        idx = torch.empty(1, wl.top_k, dtype=torch.int32, device="cuda")
        M.moe_layer(cfg, pool, dl.w_router, dl.bias, to_dev(xs[it % 3]), out, ws, topk_idx_out=idx)
        torch.cuda.synchronize()
        assert_ok(ws)
        if it % 3 in outs:
            assert torch.equal(out, outs[it % 3])
        else:
            outs[it % 3], idxs[it % 3] = out, idx.cpu().numpy()
    for s_ in range(3):
        compare_layer(wl, L, xs[s_], outs[s_], idxs[s_])
