#!/usr/bin/env python
"""MoE-layer decode benchmark on B200: tokens/s and int4 expert-weight HBM GB/s.

A step is one pass of the whole layer (quantise, route, bucket, gate/up,
requantise, down, combine with the shared expert) over one batch of the
workload: by default the single-token decode layer (d=6144, f=2048, 256 routed
experts + 1 shared, top-8, int4 experts, ~4.8 GB pool resident in HBM), one
of 100 seeded bf16 tokens per step.  The L2 cache is flushed (a 256 MiB write)
between timed steps, outside the per-step CUDA events, so the shared expert
and the router weights are read from HBM every step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun each rank runs an independent replica on its own GPU with its
own token stream (decode tokens are independent problems: weak scaling, no
collective on the data path); timing is the max over ranks.
--impl reference times the CPU oracle (plain C) on the same workload.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer decode tokens/s; int4 expert-weight HBM GB/s vs 8 TB/s peak"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", type=int, default=1, help="workload id (1 = decode T=1, the metric's config)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="time budget of the oracle CPU baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--trace", default="", help="write per-CTA phase stamps of one extra step to this JSON file")
    ap.add_argument("--n-experts", type=int, default=0,
                    help="profiling case: the same layer with fewer routed experts (smaller pool)")
    return ap.parse_args()


def metric_for(wl, workload_id):
    """The headline metric on its own workload; a labelled variant elsewhere."""
    return METRIC if workload_id == 1 else f"MoE-layer tokens/s on {wl.name}; expert-weight HBM GB/s"


def dtype_for(wl):
    return "i8*i4->i32" if wl.wbits == 4 else "i8*i2->i32"


def rank_token_sets(rank, n_sets):
    """Seeds of a rank's token stream: every replica draws its own tokens
    (rank 0's stream is the single-GPU one)."""
    return [rank * 1000 + s for s in range(n_sets)]


def max_over_ranks(ms, world, dist=None, device=None):
    """The slowest rank's time: every rank calls this (the same collective in
    the same order on all ranks) and gets the maximum."""
    if world <= 1:
        return float(ms)
    import torch
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world, steps, tokens_per_step, max_ms):
    """Tokens per second of all ranks together over the slowest rank's time."""
    return world * steps * tokens_per_step / (max_ms / 1e3)


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            pk = json.load(fh)
        return float(pk["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons during a region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.rows = []
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None
        return self

    def wait_first(self, timeout=10.0):
        t0 = time.time()
        while self.proc is not None and not self.rows and time.time() - t0 < timeout:
            time.sleep(0.02)

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append([c.strip() for c in line.split(",")])

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm = [float(r[1]) for r in self.rows if len(r) > 8 and r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in self.rows if len(r) > 8 and r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows if len(r) > 8 for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.rows)}


# ---------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline leg and the reference arm)
# ---------------------------------------------------------------------------
def oracle_decode_timer(wl, seed, token_sets, max_tokens=None):
    """Prepare the oracle on the workload: route every sampled token once,
    generate the selected experts' blobs, and return a function that runs the
    oracle layer on one token set (at most max_tokens of its tokens; timed by
    the caller)."""
    import numpy as np

    import oracle as O
    import workloads as W
    L = W.layer(wl, seed, 0)
    xs = [W.tokens(wl, seed, s).float().numpy()[:max_tokens] for s in token_sets]
    need = {wl.n_experts} if wl.has_shared else set()
    for x in xs:
        idx, _ = O.route(x, L.w_router, L.bias, wl.top_k, wl.routed_scale)
        need |= set(idx.reshape(-1).tolist())
    blobs = [None] * wl.n_blobs
    scales = [None] * wl.n_blobs
    sc = L.scales.numpy()
    for e in sorted(need):
        blobs[e] = W.expert_blob(wl, seed, 0, e).numpy()
        scales[e] = np.ascontiguousarray(sc[e])
    wr, b = L.w_router.numpy(), L.bias.numpy()

    def run(i):
        return O.layer(wl.d, wl.f, wl.n_experts, wl.top_k, wl.has_shared, wl.wbits, wl.routed_scale, blobs, scales,
                       wr, b, xs[i % len(xs)])
    return run


def cpu_baseline(wl, budget_s):
    """The oracle layer on a bounded sample: up to 16 single-token sets, or 4
    sets of at most 4 tokens for batched workloads (the oracle's per-token
    cost of the layer does not depend on T)."""
    import oracle as O
    per = min(wl.T, 4)
    n_sets = 16 if per == 1 else 4  # bounds the experts generated on the host
    run = oracle_decode_timer(wl, 0, list(range(n_sets)), max_tokens=per)
    n, t0 = 0, time.perf_counter()
    while True:
        run(n)
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s or n >= n_sets:
            break
    return {"value": n * per / el, "unit": "tokens/s", "cores": O.num_threads(), "kind": "oracle",
            "sample": f"{n} calls of {per} token(s) of {wl.name}, full layer, {el:.1f} s of CPU work"}


def reference_arm(args, wl):
    import oracle as O
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    K, Wm = args.steps, args.warmup
    # a bounded sample per step: the whole token for decode, at most 4 tokens
    # of a batched workload (the oracle's per-token cost does not depend on T)
    per = min(wl.T, 4)
    run = oracle_decode_timer(wl, 0, list(range(min(100, K + Wm))), max_tokens=per)
    for i in range(Wm):
        run(i)
    t0 = time.perf_counter()
    for i in range(K):
        run(Wm + i)
    el = time.perf_counter() - t0
    v = K * per / el
    line = {"impl": "reference", "metric": metric_for(wl, args.workload), "value": v, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": K, "warmup": Wm, "ms_per_step": 1e3 * el / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": dtype_for(wl), "data": "synthetic",
            "config": {"workload": wl.name, "T": wl.T, "d": wl.d, "f": wl.f, "experts": wl.n_experts,
                       "shared": wl.has_shared, "top_k": wl.top_k, "wbits": wl.wbits},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": O.num_threads(), "kind": "oracle",
                             "sample": f"{K} timed steps of {per} token(s) of {wl.name}, full layer"},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
TRACE_NAMES = {0: "start", 1: "quantised", 2: "router_done", 3: "shared_gate_up_done", 4: "grid_barrier",
               5: "routing_done", 6: "routed_gate_up_done", 7: "first_down_staged", 8: "down_done",
               9: "cons_wait_full_total", 10: "prod_wait_empty_total", 11: "topk_done",
               12: "prod_pre_routing_issued", 13: "prod_routing_received", 14: "prod_all_issued",
               15: "prod_drained", 16: "designated_h_row_complete", 17: "designated_codes_written",
               20: "first_down_codes_seen", 21: "last_down_unit_done"}


def write_trace(path, M, cfg, pool, dl, xbuf, out, ws, dev, flush_l2):
    """One extra step of the single-launch path with the phase trace on; writes
    per-phase stamps (us after the earliest CTA start) as min/median/max over CTAs."""
    import torch
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    tr = torch.zeros(sms, 32, dtype=torch.int64, device=dev)
    o = M.MoeLayerOpts()
    o.trace = tr.data_ptr()
    flush_l2(0)
    M.moe_layer(cfg, pool, dl.w_router, dl.bias, xbuf, out, ws, opts=o)
    torch.cuda.synchronize()
    t = tr.cpu().numpy().astype("float64")
    t0 = t[:, 0].min()
    rec = {}
    for i, name in TRACE_NAMES.items():
        col = t[:, i]
        col = col[col > 0]
        if col.size:
            v = (col - (0 if name.endswith("_total") else t0)) / 1e3
            rec[name] = {"min": float(v.min()), "median": float(sorted(v)[len(v) // 2]), "max": float(v.max())}
    raw = ((t - t0) / 1e3).round(3).tolist()
    with open(path, "w") as fh:
        json.dump({"us_after_first_cta_start": rec, "ctas": int(sms), "raw_us": raw}, fh)


def gpu_arm(args, wl):
    import numpy as np
    import torch
    import torch.distributed as dist

    import expert_ffn_router_b200 as M
    import workloads as W

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    K, Wm = args.steps, args.warmup
    T = wl.T
    cfg = M.config(wl.d, wl.f, wl.n_experts, wl.top_k, wl.has_shared, wl.wbits, wl.routed_scale)
    L = W.layer(wl, 0, 0)
    dl = W.device_layer(wl, 0, 0, dev, host=L)
    pool = M.make_pool(dl.pool_w, dl.pool_s)
    n_sets = wl.n_token_sets
    # every rank draws its own token stream
    toks = torch.stack([W.tokens(wl, 0, s) for s in rank_token_sets(rank, n_sets)]).to(dev)  # [n_sets][T][d]
    xbuf = torch.empty(T, wl.d, dtype=toks.dtype, device=dev)
    out = torch.empty(T, wl.d, device=dev)
    idx = torch.empty(T, wl.top_k, dtype=torch.int32, device=dev)
    ws = M.workspace(cfg, T, dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_rd = torch.ones(256 << 18, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)

    def flush_l2(i):
        # write 256 MiB (evicts the step's lines), then read another 256 MiB so
        # the dirty lines are written back here, not inside the next timed step
        flush.fill_(i & 0xFF)
        torch.sum(flush_rd, dim=0, out=sink)
    stream = torch.cuda.current_stream()
    n_ev = K
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n_ev)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
    for i in range(n_ev):  # torch creates CUDA events lazily: record once so the handles exist
        for e in ev[i] + [ends[i]]:
            e.record(stream)
    opts = [M.MoeLayerOpts() for _ in range(n_ev)]
    for i in range(n_ev):
        for j in range(4):
            opts[i].events[j] = ev[i][j].cuda_event
            assert opts[i].events[j], "CUDA event handle not created"
    idx_log = torch.empty(K, T, wl.top_k, dtype=torch.int32, device=dev)

    def step(i, o=None, log=None):
        xbuf.copy_(toks[i % n_sets])
        M.moe_layer(cfg, pool, dl.w_router, dl.bias, xbuf, out, ws, topk_idx_out=log, opts=o)

    for i in range(Wm):
        flush_l2(i)
        step(i)
    assert M.moe_poll_status(ws) == M.MOE_OK
    barrier()
    torch.cuda.synchronize()
    launches = 0
    with Clocks(local) as clk:
        clk.wait_first()
        for i in range(K):
            flush_l2(i)
            xbuf.copy_(toks[(Wm + i) % n_sets])
            M.moe_layer(cfg, pool, dl.w_router, dl.bias, xbuf, out, ws, topk_idx_out=idx_log[i], opts=opts[i])
            ends[i].record(stream)
            launches += opts[i].n_launches
        torch.cuda.synchronize()
    barrier()
    step_ms = [ev[i][0].elapsed_time(ev[i][3]) for i in range(K)]
    # the single-launch decode path records only events [0] and [3]
    phased = opts[0].path_ran != M.MOE_PATH_DECODE
    route_ms = [ev[i][0].elapsed_time(ev[i][1]) if phased else 0.0 for i in range(K)]
    gu_ms = [ev[i][1].elapsed_time(ev[i][2]) if phased else 0.0 for i in range(K)]
    dn_ms = [ev[i][2].elapsed_time(ev[i][3]) if phased else 0.0 for i in range(K)]
    total_ms = sum(step_ms)
    assert M.moe_poll_status(ws) == M.MOE_OK

    # unique experts per step (dedupe: each selected expert is read once)
    il = idx_log.cpu().numpy()
    uniq = [len(set(il[i].reshape(-1).tolist())) + wl.has_shared for i in range(K)]
    gu_bytes_e = 2 * wl.f * wl.d * wl.wbits // 8 + 2 * wl.f * 4
    dn_bytes_e = wl.d * wl.f * wl.wbits // 8 + wl.d * 4
    exp_bytes = sum(u * (gu_bytes_e + dn_bytes_e) for u in uniq)

    max_ms = max_over_ranks(total_ms, world, dist, dev)

    e2e = None
    if not args.no_e2e:
        hx = torch.empty(n_sets, T, wl.d, dtype=toks.dtype).pin_memory()
        hx.copy_(toks.cpu())
        hout = torch.empty(T, wl.d).pin_memory()
        e_s = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
        e_e = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
        barrier()
        torch.cuda.synchronize()
        for i in range(K):
            flush_l2(i)
            e_s[i].record(stream)
            xbuf.copy_(hx[i % n_sets], non_blocking=True)
            M.moe_layer(cfg, pool, dl.w_router, dl.bias, xbuf, out, ws)
            hout.copy_(out, non_blocking=True)
            e_e[i].record(stream)
        torch.cuda.synchronize()
        barrier()
        e2e_ms = max_over_ranks(sum(e_s[i].elapsed_time(e_e[i]) for i in range(K)), world, dist, dev)
        e2e = {"value": whole_job_rate(world, K, T, e2e_ms), "unit": "tokens/s",
               "h2d_bytes_per_step": T * wl.d * toks.element_size(), "d2h_bytes_per_step": T * wl.d * 4,
               "api": "expert_ffn_router_b200.moe_layer (libmoe.so moe_layer), pinned host buffers"}

    ran = opts[0].path_ran
    single = ran == M.MOE_PATH_DECODE
    router_bytes = wl.n_experts * wl.d * 4
    if args.trace and rank == 0:
        write_trace(args.trace, M, cfg, pool, dl, xbuf, out, ws, dev, flush_l2)
    if rank == 0:
        hbm, which = peaks()
        if single:  # one kernel does the whole layer: its bytes are every expert's plus the router's
            kname = "k_decode"
            k_avg_s = statistics.mean(step_ms) / 1e3
            k_alg = statistics.mean(u * (gu_bytes_e + dn_bytes_e) for u in uniq) + router_bytes
        else:  # the gate/up kernel: every unique expert's gate and up rows once
            kname = "k_tc<gate/up>" if ran == M.MOE_PATH_TC else "k_gate_up"
            k_avg_s = statistics.mean(gu_ms) / 1e3
            k_alg = statistics.mean(u * gu_bytes_e for u in uniq)
        achieved = k_alg / k_avg_s / 1e9
        traffic = None
        try:  # ncu DRAM bytes of this kernel and workload, if taken on the current sources
            with open(os.path.join(ROOT, "profiles", "traffic.json")) as fh:
                recs = json.load(fh).get("records", [])
            import importlib.util
            spec = importlib.util.spec_from_file_location("_moe_build", os.path.join(ROOT, "expert_ffn_router_b200",
                                                                                     "build.py"))
            B = importlib.util.module_from_spec(spec)
            spec.loader.exec_module(B)
            h = B.source_hash()
            for tr in recs:
                if tr.get("source_hash") == h and tr.get("workload") == wl.name and tr.get("kernel") == kname:
                    traffic = tr.get("bytes_per_launch")
        except Exception:
            traffic = None
        value = whole_job_rate(world, K, T, max_ms)
        exp_gbs = exp_bytes / (total_ms / 1e3) / 1e9
        line = {
            "metric": metric_for(wl, args.workload),
            "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": Wm,
            "ms_per_step": max_ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": dtype_for(wl), "data": "synthetic",
            "config": {"workload": wl.name, "T": T, "d": wl.d, "f": wl.f, "experts": wl.n_experts,
                       "shared": wl.has_shared, "top_k": wl.top_k, "wbits": wl.wbits,
                       "pool_gb": wl.pool_bytes / 1e9, "token_sets": n_sets,
                       "l2": "flushed between timed steps (256 MiB write, then 256 MiB read), outside the per-step events",
                       "parallelism": f"replicas{world}"},
            "expert_weight_gbs": exp_gbs, "expert_weight_frac_of_8tbs": exp_gbs / NOMINAL_HBM_GBS,
            "expert_weight_frac_of_measured": exp_gbs / hbm, "unique_experts_per_step": statistics.mean(uniq),
            "path": {M.MOE_PATH_DECODE: "decode", M.MOE_PATH_MULTI: "multi", M.MOE_PATH_TC: "tensor_core"}.get(ran),
            "phase_ms": ({"layer_single_launch": statistics.mean(step_ms)} if single else
                         {"route": statistics.mean(route_ms), "gate_up": statistics.mean(gu_ms),
                          "down_combine": statistics.mean(dn_ms)}),
            "roofline": {"kernel": kname, "bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                         "frac": achieved / hbm, "peak_source": which, "traffic": traffic,
                         "alg_bytes_per_launch": k_alg},
            "gpu_launches": launches,
            "clocks": clk.summary(),
        }
        if e2e is not None:
            line["e2e"] = e2e
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(wl, args.cpu_seconds)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def main():
    args = parse()
    import workloads as W
    wl = W.workload(args.workload)
    if args.n_experts:
        wl = wl.replace(n_experts=args.n_experts, name=f"{wl.name}_e{args.n_experts}")
    if args.impl == "reference":
        reference_arm(args, wl)
    else:
        gpu_arm(args, wl)


if __name__ == "__main__":
    main()
