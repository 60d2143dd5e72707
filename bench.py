#!/usr/bin/env python
"""MoE-layer decode benchmark on B200: tokens/s and int4 expert-weight HBM GB/s.

A step is one pass of the whole workload over one batch of its tokens: every
layer's quantise, route, bucket, gate/up, requantise, down and combine with
the shared expert.  By default that is the single-token decode layer (d=6144,
f=2048, 256 routed experts + 1 shared, top-8, int4 experts, ~4.8 GB pool
resident in HBM), one of 100 seeded bf16 tokens per step.  The stacked
workloads (--workload 2: 4 tokens through 8 int4 layers, 38.7 GB; --workload
4: 64 tokens through 24 int2 layers with Zipf-skewed routing, 58.2 GB) hold
every layer's pool resident and run parameter-free RMSNorm -> layer ->
residual add through all layers per step.  The L2 cache is flushed (a 256 MiB
write, then a 256 MiB read) between timed steps, outside the per-step CUDA
events, so every step reads its weights from HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload 1|2|3|4]

Under torchrun each rank runs an independent replica on its own GPU with its
own token stream (decode tokens are independent problems: weak scaling, no
collective on the data path); timing is the max over ranks.
--impl reference times the CPU oracle (plain C) on the same workload.
"""
import argparse
import json
import os
import platform
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


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", type=int, default=1, help="workload id (1 = decode T=1, the metric's config)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="time budget of the oracle CPU baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--trace", default="", help="write per-CTA phase stamps of one extra step to this JSON file")
    ap.add_argument("--n-experts", type=int, default=0,
                    help="profiling case: the same layer with fewer routed experts (smaller pool)")
    ap.add_argument("--layers", type=int, default=0, help="profiling case: the first N layers of a stack")
    ap.add_argument("--cache-slots", type=int, default=0,
                    help="supplementary case: the layer's pool in pinned host memory behind an HBM expert cache "
                         "of this many slots (moe_cache_fetch); reports hit rate and host->device bytes per token")
    ap.add_argument("--topp", type=float, default=0.0,
                    help="supplementary case: the router's TOPK/TOPP truncation at this threshold "
                         "(moe_config.topp; fewer experts per token)")
    ap.add_argument("--tokens", type=int, default=0,
                    help="supplementary case: the workload with this many tokens per step (e.g. prefill at 8192)")
    ap.add_argument("--wbits", type=int, choices=[2, 4, 8], default=0,
                    help="supplementary case: the workload with expert codes of this width (int8: one code per byte)")
    ap.add_argument("--path", choices=["auto", "multi", "decode", "tc"], default="auto",
                    help="comparison case: force one of the library's layer paths (moe_layer_opts.path)")
    ap.add_argument("--int8-peak", action="store_true",
                    help="measure the dense int8 tensor-core peak (torch._int_mm at 8192^3) and write it to "
                         "profiles/int8_peak.json")
    return ap.parse_args(argv)


def metric_for(wl, workload_id):
    """The headline metric on its own workload, unmodified; a labelled variant
    elsewhere."""
    import workloads as W
    if workload_id == 1 and wl.name == W.workload(1).name:
        return METRIC
    return f"MoE-layer tokens/s on {wl.name}; expert-weight HBM GB/s"


def dtype_for(wl):
    return f"i8*i{wl.wbits}->i32"


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


def expert_bytes(wl):
    """Bytes one expert's gate/up and down rows (codes + fp32 row scales) take."""
    gu = 2 * wl.f * wl.d * wl.wbits // 8 + 2 * wl.f * 4
    dn = wl.d * wl.f * wl.wbits // 8 + wl.d * 4
    return gu, dn


def percentiles(v):
    s = sorted(v)
    n = len(s)
    return {"median": s[n // 2], "p10": s[n // 10], "p90": s[min(n - 1, (9 * n) // 10)], "min": s[0],
            "max": s[-1]}


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            pk = json.load(fh)
        return float(pk["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def cpu_model():
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or "unknown"


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
                                          "--format=csv,noheader,nounits", "-lms", "20"],
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
class OracleRunner:
    """The CPU oracle on a workload: one layer per call for single-layer
    workloads, the whole stack (RMSNorm -> layer -> residual) for stacked
    ones.  Expert blobs are generated on the host, outside the timed part;
    ``run(x)`` returns the oracle's compute seconds for the tokens x."""

    def __init__(self, wl, n_layers):
        import oracle as O
        import workloads as W
        self.O, self.W, self.wl = O, W, wl
        self.n_layers = n_layers
        self.layers = [W.layer(wl, 0, l) for l in range(n_layers)]
        self.cache = {}
        self.cache_bytes = 3e9

    def _blobs(self, l, idx):
        wl, W = self.wl, self.W
        need = (set(idx.reshape(-1).tolist()) - {-1}) | ({wl.n_experts} if wl.has_shared else set())
        blobs, scales = [None] * wl.n_blobs, [None] * wl.n_blobs
        sc = self.layers[l].scales.numpy()
        if len(self.cache) * wl.blob_bytes > self.cache_bytes:
            self.cache.clear()  # bounds host memory on stacks; regenerating is not timed
        for e in need:
            if (l, e) not in self.cache:
                self.cache[(l, e)] = W.expert_blob(wl, 0, l, e).numpy()
            blobs[e] = self.cache[(l, e)]
            scales[e] = sc[e].copy()
        return blobs, scales

    def run(self, x):
        import numpy as np
        O, wl = self.O, self.wl
        stack = self.n_layers > 1 or wl.residual
        xr = np.asarray(x, np.float64)
        spent = 0.0
        for l in range(self.n_layers):
            L = self.layers[l]
            x_in = O.rmsnorm(xr) if stack else np.asarray(x, np.float32)
            idx, _ = O.route(x_in, L.w_router, L.bias, wl.top_k, wl.routed_scale, topp=wl.topp)
            blobs, scales = self._blobs(l, idx)  # generation: not timed
            t0 = time.perf_counter()
            r = O.layer(wl.d, wl.f, wl.n_experts, wl.top_k, wl.has_shared, wl.wbits, wl.routed_scale, blobs, scales,
                        L.w_router, L.bias, x_in, topp=wl.topp)
            spent += time.perf_counter() - t0
            xr = xr + r["out"] if stack else r["out"]
        return spent


def cpu_baseline(wl, budget_s, n_layers):
    """The oracle on a bounded sample of the workload: single tokens (one per
    call) through the whole workload (every layer of a stack), all host cores,
    then the same on one core; the oracle's cost per token does not depend on
    the batch size (it computes each token's experts on their own)."""
    import oracle as O
    import workloads as W
    run = OracleRunner(wl, n_layers)
    n_sets = wl.n_token_sets if wl.n_token_sets > 1 else 4

    def one(i):
        s, t = divmod(i, wl.T)
        return run.run(W.tokens(wl, 0, s % n_sets).float().numpy()[t:t + 1])

    def timed(limit_calls, limit_s):
        n, el = 0, 0.0
        while n < limit_calls and el < limit_s:
            el += one(n)
            n += 1
        return n, el

    cores = O.num_threads()
    n, el = timed(16, budget_s)
    res = {"value": n / el, "unit": "tokens/s", "cores": cores, "kind": "oracle", "cpu_model": cpu_model(),
           "sample": f"{n} single-token calls of {wl.name} through {n_layers} layer(s), {el:.2f} s of oracle "
                     f"compute on {cores} threads (expert generation on the host not timed)"}
    O.set_num_threads(1)
    try:
        n1, el1 = timed(4, budget_s / 3)
    finally:
        O.set_num_threads(cores)
    res["single_thread"] = {"value": n1 / el1, "unit": "tokens/s", "cores": 1,
                            "sample": f"{n1} single-token calls, {el1:.2f} s on one thread"}
    return res


def reference_arm(args, wl):
    import oracle as O
    import workloads as W
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    K, Wm = args.steps, args.warmup
    n_layers = getattr(args, "layers", 0) or wl.n_layers
    run = OracleRunner(wl, n_layers)
    # a bounded sample per step: one token of the step's batch through every
    # layer (the oracle's cost per token does not depend on the batch size)
    n_sets = min(100, wl.n_token_sets) if wl.n_token_sets > 1 else 2
    xs = [W.tokens(wl, 0, s % n_sets).float().numpy()[:1] for s in range(min(K + Wm, n_sets))]
    for i in range(Wm):
        run.run(xs[i % len(xs)])
    el = 0.0
    for i in range(K):
        el += run.run(xs[(Wm + i) % len(xs)])
    v = K / el
    line = {"impl": "reference", "metric": metric_for(wl, args.workload), "value": v, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": K, "warmup": Wm, "ms_per_step": 1e3 * el / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": dtype_for(wl), "data": "synthetic",
            "config": {"workload": wl.name, "T": wl.T, "d": wl.d, "f": wl.f, "experts": wl.n_experts,
                       "shared": wl.has_shared, "top_k": wl.top_k, "wbits": wl.wbits, "layers": n_layers},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": O.num_threads(), "kind": "oracle",
                             "cpu_model": cpu_model(),
                             "sample": f"{K} timed steps of 1 token of {wl.name} through {n_layers} layer(s) "
                                       f"(expert generation on the host not timed)"},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
TRACE_NAMES = {0: "start", 1: "quantised", 2: "router_done", 3: "shared_gate_up_done", 4: "grid_barrier",
               5: "routing_done", 6: "routed_gate_up_done", 7: "designated_requant_done", 8: "down_done",
               9: "cons_wait_full_total", 10: "prod_wait_empty_total", 11: "topk_done",
               12: "prod_pre_routing_issued", 13: "prod_routing_received", 14: "prod_all_issued",
               15: "prod_drained", 16: "designated_h_row_complete", 17: "designated_codes_written",
               18: "topk_values_loaded", 20: "all_codes_staged", 21: "last_down_unit_done",
               22: "first_down_unit_done"}


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


def traffic_record(kname, wl):
    """ncu DRAM bytes per launch of this kernel and workload, if recorded on
    the current sources (profiles/traffic.json), else None."""
    try:
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
                return tr.get("bytes_per_launch")
    except Exception:
        pass
    return None


def gpu_arm(args, wl):
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
    n_layers = args.layers or wl.n_layers
    stack = n_layers > 1 or wl.residual
    cfg = M.config(wl.d, wl.f, wl.n_experts, wl.top_k, wl.has_shared, wl.wbits, wl.routed_scale,
                   topp=wl.topp)
    layers = [W.device_layer(wl, 0, l, dev) for l in range(n_layers)]
    pools = [M.make_pool(dl.pool_w, dl.pool_s) for dl in layers]
    n_sets = wl.n_token_sets if wl.n_token_sets > 1 else 4
    # every rank draws its own token stream
    toks = torch.stack([W.tokens(wl, 0, s) for s in rank_token_sets(rank, n_sets)]).to(dev)  # [n_sets][T][d]
    xbuf = torch.empty(T, wl.d, dtype=toks.dtype, device=dev)
    out = torch.empty(T, wl.d, device=dev)       # single layer: the output; stack: the residual stream
    x_in = torch.empty(T, wl.d, device=dev)      # stack: the normalised layer input
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

    plain = [M.MoeLayerOpts() for _ in range(n_layers)]  # the chosen path, no events
    for o in plain:
        o.path = {"auto": M.MOE_PATH_AUTO, "multi": M.MOE_PATH_MULTI, "decode": M.MOE_PATH_DECODE,
                  "tc": M.MOE_PATH_TC}[getattr(args, "path", "auto")]

    def run_step(opts_row, idx_row, x_src=None):
        """One step on the stream: every layer of the workload on xbuf."""
        if opts_row is None:
            opts_row = plain
        src = xbuf if x_src is None else x_src
        if not stack:
            M.moe_layer(cfg, pools[0], layers[0].w_router, layers[0].bias, src, out, ws,
                        topk_idx_out=None if idx_row is None else idx_row[0], opts=opts_row[0])
            return
        M.moe_rmsnorm(src, x_in, 1e-6, x_copy=out)
        for l in range(n_layers):
            if l > 0:
                M.moe_rmsnorm(out, x_in, 1e-6)
            M.moe_layer(cfg, pools[l], layers[l].w_router, layers[l].bias, x_in, out, ws, accumulate=True,
                        topk_idx_out=None if idx_row is None else idx_row[l], opts=opts_row[l])

    # per step: events around the step, and each layer call's phase events
    st_ev = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    en_ev = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev = [[[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n_layers)] for _ in range(K)]
    for i in range(K):  # torch creates CUDA events lazily: record once so the handles exist
        for e in [st_ev[i], en_ev[i]] + [e for row in ev[i] for e in row]:
            e.record(stream)
    path_id = {"auto": M.MOE_PATH_AUTO, "multi": M.MOE_PATH_MULTI, "decode": M.MOE_PATH_DECODE,
               "tc": M.MOE_PATH_TC}[getattr(args, "path", "auto")]
    opts = [[M.MoeLayerOpts() for _ in range(n_layers)] for _ in range(K)]
    for i in range(K):
        for l in range(n_layers):
            opts[i][l].path = path_id
            for j in range(4):
                opts[i][l].events[j] = ev[i][l][j].cuda_event
                assert opts[i][l].events[j], "CUDA event handle not created"
    idx_log = torch.empty(K, n_layers, T, wl.top_k, dtype=torch.int32, device=dev)

    for i in range(Wm):
        flush_l2(i)
        xbuf.copy_(toks[i % n_sets])
        run_step(None, None)
    assert M.moe_poll_status(ws) == M.MOE_OK
    barrier()
    torch.cuda.synchronize()
    launches = 0
    with Clocks(local) as clk:
        clk.wait_first()
        for i in range(K):
            flush_l2(i)
            xbuf.copy_(toks[(Wm + i) % n_sets])
            if stack:
                st_ev[i].record(stream)
            run_step(opts[i], idx_log[i])
            if stack:
                en_ev[i].record(stream)
            launches += sum(o.n_launches for o in opts[i]) + (n_layers if stack else 0)  # + the RMSNorms
        torch.cuda.synchronize()
    barrier()
    ran = opts[0][0].path_ran
    single = ran == M.MOE_PATH_DECODE
    # a single-layer step is the layer call itself (its events [0] and [3]
    # bracket the launches); a stack's step adds the RMSNorms between layers
    if stack:
        step_ms = [st_ev[i].elapsed_time(en_ev[i]) for i in range(K)]
    else:
        step_ms = [ev[i][0][0].elapsed_time(ev[i][0][3]) for i in range(K)]
    # the dominant kernel of each layer call: the single-launch decode kernel
    # (events [0] -> [3]), else the gate/up kernel (events [1] -> [2])
    if single:
        kern_ms = [ev[i][l][0].elapsed_time(ev[i][l][3]) for i in range(K) for l in range(n_layers)]
    else:
        kern_ms = [ev[i][l][1].elapsed_time(ev[i][l][2]) for i in range(K) for l in range(n_layers)]
    phase = None
    if not single:
        phase = {"route": statistics.mean(ev[i][l][0].elapsed_time(ev[i][l][1]) for i in range(K)
                                          for l in range(n_layers)),
                 "gate_up": statistics.mean(kern_ms),
                 "down_combine": statistics.mean(ev[i][l][2].elapsed_time(ev[i][l][3]) for i in range(K)
                                                 for l in range(n_layers))}
    total_ms = sum(step_ms)
    assert M.moe_poll_status(ws) == M.MOE_OK

    # unique experts per layer call (dedupe: each selected expert is read once)
    il = idx_log.cpu().numpy()
    uniq = [len(set(il[i][l].reshape(-1).tolist()) - {-1}) + wl.has_shared  # -1: a slot TOPP dropped
            for i in range(K) for l in range(n_layers)]
    gu_b, dn_b = expert_bytes(wl)
    step_exp_bytes = sum(u * (gu_b + dn_b) for u in uniq) / K  # counted expert bytes per step
    max_ms = max_over_ranks(total_ms, world, dist, dev)

    e2e = None
    if not args.no_e2e:
        host_io = None
        if not stack and T <= 8:
            # decode-sized single layer: the call reads the token from, and
            # writes the output to, pinned host memory itself
            o_io = M.MoeLayerOpts()
            o_io.path = path_id
            o_io.io_host = M.MOE_IO_X_HOST | M.MOE_IO_OUT_HOST

            def host_io(xh, outh):
                M.moe_layer(cfg, pools[0], layers[0].w_router, layers[0].bias, xh, outh, ws, opts=o_io)
        e2e = e2e_arm(args, wl, M, torch, dist, world, dev, stream, toks, xbuf, out, run_step, host_io, flush_l2, barrier,
                      n_sets)

    if args.trace and rank == 0 and single and not stack:
        write_trace(args.trace, M, cfg, pools[0], layers[0], xbuf, out, ws, dev, flush_l2)
    if rank == 0:
        hbm, which = peaks()
        if single:
            kname = "k_decode"
            k_alg = statistics.mean(u * (gu_b + dn_b) for u in uniq)
        else:
            kname = "k_tc<gate/up>" if ran == M.MOE_PATH_TC else "k_gate_up"
            k_alg = statistics.mean(u * gu_b for u in uniq)
        k_avg_s = statistics.mean(kern_ms) / 1e3
        achieved = k_alg / k_avg_s / 1e9
        value = whole_job_rate(world, K, T, max_ms)
        exp_gbs = step_exp_bytes * K / (total_ms / 1e3) / 1e9
        router_bytes = wl.n_experts * wl.d * 4
        line = {
            "metric": metric_for(wl, args.workload),
            "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": Wm,
            "ms_per_step": max_ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": dtype_for(wl), "data": "synthetic",
            "config": {"workload": wl.name, "T": T, "d": wl.d, "f": wl.f, "experts": wl.n_experts,
                       "shared": wl.has_shared, "top_k": wl.top_k, "wbits": wl.wbits, "layers": n_layers,
                       "pool_gb": wl.pool_bytes * n_layers / 1e9, "token_sets": n_sets,
                       "l2": "flushed between timed steps (256 MiB write, then 256 MiB read), outside the per-step events",
                       "parallelism": f"replicas{world}"},
            "step_ms": percentiles(step_ms),
            "expert_weight_gbs": exp_gbs, "expert_weight_frac_of_8tbs": exp_gbs / NOMINAL_HBM_GBS,
            "expert_weight_frac_of_peak": exp_gbs / hbm,
            "unique_experts_per_layer": statistics.mean(uniq) - wl.has_shared,
            "counted_expert_bytes_per_step": step_exp_bytes,
            "router_bytes_per_layer": router_bytes,
            "path": {M.MOE_PATH_DECODE: "decode", M.MOE_PATH_MULTI: "multi", M.MOE_PATH_TC: "tensor_core"}.get(ran),
            "roofline": {"kernel": kname, "bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                         "frac": achieved / hbm, "peak_source": which, "traffic": traffic_record(kname, wl),
                         "alg_bytes_per_launch": k_alg, "launch_ms": percentiles(kern_ms),
                         "alg_bytes": "expert bytes (codes + row scales) of the unique experts selected in the "
                                      "call plus the shared expert; router weights excluded"},
            "gpu_launches": launches,
            "clocks": clk.summary(),
        }
        if phase:
            line["phase_ms"] = phase
        if ran == M.MOE_PATH_TC:  # the gate/up GEMM against the measured int8 tensor peak
            ops = 2.0 * 2 * wl.f * wl.d * T * (wl.top_k + wl.has_shared)
            tensor = {"kernel": kname, "int_ops_per_launch": ops, "achieved_tops": ops / k_avg_s / 1e12}
            try:
                with open(os.path.join(ROOT, "profiles", "int8_peak.json")) as fh:
                    pk = json.load(fh)
                tensor["peak_tops"] = pk["int8_tops_burst"]
                tensor["frac"] = tensor["achieved_tops"] / pk["int8_tops_burst"]
                tensor["peak_source"] = "measured (profiles/int8_peak.json, burst)"
            except Exception:
                tensor["peak_tops"], tensor["frac"], tensor["peak_source"] = None, None, "not measured"
            line["tensor"] = tensor
        if e2e is not None:
            line["e2e"] = e2e
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(wl, args.cpu_seconds, n_layers)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def e2e_arm(args, wl, M, torch, dist, world, dev, stream, toks, xbuf, out, run_step, host_io, flush_l2, barrier,
            n_sets):
    """The same workload through the public API from pinned host buffers,
    inside the step's CUDA events: with `host_io` (a single decode-sized layer)
    the call itself reads the step's tokens from pinned host memory and writes
    the output rows into pinned host memory (moe_layer_opts.io_host); otherwise
    each step copies its tokens host -> device, runs every layer, and copies the
    result back.  Also a host-clocked loop that waits for each step's result
    before starting the next, as a decode loop consumes its output."""
    K, T = args.steps, wl.T
    hx = torch.empty(n_sets, T, wl.d, dtype=toks.dtype).pin_memory()
    hx.copy_(toks.cpu())
    hout = torch.empty(T, wl.d).pin_memory()
    in_bytes, out_bytes = T * wl.d * toks.element_size(), T * wl.d * 4
    if host_io is not None:
        e_s = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
        e_e = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
        for i in range(args.warmup):  # the staging kernel's first launch loads its module
            flush_l2(i)
            host_io(hx[i % n_sets], hout)
        barrier()
        torch.cuda.synchronize()
        for i in range(K):
            flush_l2(i)
            e_s[i].record(stream)
            host_io(hx[i % n_sets], hout)
            e_e[i].record(stream)
        torch.cuda.synchronize()
        barrier()
        steps_ms = [e_s[i].elapsed_time(e_e[i]) for i in range(K)]
        e2e_ms = max_over_ranks(sum(steps_ms), world, dist, dev)
        n_host = min(K, 200)
        wall = []
        for i in range(n_host):
            flush_l2(i)
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            host_io(hx[i % n_sets], hout)
            torch.cuda.synchronize()
            wall.append(time.perf_counter() - t0)
        wall_ms = statistics.median(wall) * 1e3
        return {"value": whole_job_rate(world, K, T, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": in_bytes, "d2h_bytes_per_step": out_bytes,
                "api": "expert_ffn_router_b200.moe_layer (libmoe.so moe_layer_ex) with io_host = MOE_IO_X_HOST | "
                       "MOE_IO_OUT_HOST: the call copies the token from pinned host memory with a staging kernel "
                       "and its kernels write the output rows into pinned host memory",
                "median_ms": {"call_with_host_io": statistics.median(steps_ms)},
                "host_loop": {"value": T / (wall_ms / 1e3), "unit": "tokens/s", "median_ms_per_step": wall_ms,
                              "steps": n_host,
                              "how": "wall clock per step from the call to its result being on the host, stream "
                                     "synchronised every step (L2 flushed before each step, not timed)"}}
    e_s = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    e_k0 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    e_k1 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    e_e = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    barrier()
    torch.cuda.synchronize()
    for i in range(K):
        flush_l2(i)
        e_s[i].record(stream)
        xbuf.copy_(hx[i % n_sets], non_blocking=True)
        e_k0[i].record(stream)
        run_step(None, None)
        e_k1[i].record(stream)
        hout.copy_(out, non_blocking=True)
        e_e[i].record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(sum(e_s[i].elapsed_time(e_e[i]) for i in range(K)), world, dist, dev)
    h2d = statistics.median(e_s[i].elapsed_time(e_k0[i]) for i in range(K))
    layer = statistics.median(e_k0[i].elapsed_time(e_k1[i]) for i in range(K))
    d2h = statistics.median(e_k1[i].elapsed_time(e_e[i]) for i in range(K))
    # host-clocked loop: one step at a time, waiting for its result
    n_host = min(K, 200)
    wall = []
    for i in range(n_host):
        flush_l2(i)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        xbuf.copy_(hx[i % n_sets], non_blocking=True)
        run_step(None, None)
        hout.copy_(out, non_blocking=True)
        torch.cuda.synchronize()
        wall.append(time.perf_counter() - t0)
    wall_ms = statistics.median(wall) * 1e3
    return {"value": whole_job_rate(world, K, T, e2e_ms), "unit": "tokens/s",
            "h2d_bytes_per_step": in_bytes, "d2h_bytes_per_step": out_bytes,
            "api": "expert_ffn_router_b200.moe_layer (libmoe.so moe_layer), pinned host buffers",
            "median_ms": {"h2d_copy": h2d, "layers": layer, "d2h_copy": d2h},
            "host_loop": {"value": T / (wall_ms / 1e3), "unit": "tokens/s", "median_ms_per_step": wall_ms,
                          "steps": n_host,
                          "how": "wall clock per step from the H2D copy to the D2H result being on the host, "
                                 "stream synchronised every step (L2 flushed before each step, not timed)"}}


def cache_arm(args, wl):
    """One layer, T tokens per call, with its pool in pinned host memory behind
    an HBM expert cache: each step routes, copies the indices to the host,
    fetches the missing experts (one DMA copy each) and runs the layer on the
    cached pool; timed by the host clock per synchronised step (the fetch
    needs the routing on the host).  Reports tokens/s, the hit rate and the
    host -> device bytes per token."""
    import torch
    import expert_ffn_router_b200 as M
    import workloads as W
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    K, Wm, T = args.steps, args.warmup, wl.T
    cfg = M.config(wl.d, wl.f, wl.n_experts, wl.top_k, wl.has_shared, wl.wbits, wl.routed_scale, topp=wl.topp)
    dl = W.device_layer(wl, 0, 0, dev)
    host_w = dl.pool_w.cpu().pin_memory()
    del dl.pool_w  # only the cache's slots stay in HBM
    torch.cuda.empty_cache()
    cache = M.ExpertCache(cfg, host_w, dl.pool_s, args.cache_slots, dev)
    n_sets = wl.n_token_sets if wl.n_token_sets > 1 else 4
    toks = torch.stack([W.tokens(wl, 0, s) for s in range(n_sets)]).to(dev)
    ws = M.workspace(cfg, T, dev)
    out = torch.empty(T, wl.d, device=dev)
    idx = torch.empty(T, wl.top_k, dtype=torch.int32, device=dev)
    w = torch.empty(T, wl.top_k, device=dev)
    idx_h = torch.empty(T, wl.top_k, dtype=torch.int32).pin_memory()

    def step(i):
        x = toks[i % n_sets]
        M.moe_route(cfg, x, dl.w_router, dl.bias, idx, w, ws)
        idx_h.copy_(idx, non_blocking=True)
        torch.cuda.synchronize()
        st = cache.fetch(idx_h)
        M.moe_layer(cfg, cache.pool, dl.w_router, dl.bias, x, out, ws)
        torch.cuda.synchronize()
        return st

    for i in range(Wm):
        step(i)
    wall, hits, misses, nbytes = [], 0, 0, 0
    for i in range(K):
        t0 = time.perf_counter()
        st = step(Wm + i)
        wall.append(time.perf_counter() - t0)
        hits, misses, nbytes = hits + st.hits, misses + st.misses, nbytes + st.bytes
    assert M.moe_poll_status(ws) == M.MOE_OK
    total = sum(wall)
    line = {"metric": "MoE-layer decode tokens/s with an HBM expert cache (pool in pinned host memory)",
            "value": K * T / total, "unit": "tokens/s", "n_gpus": 1, "steps": K, "warmup": Wm,
            "ms_per_step": 1e3 * total / K, "step_ms_median": 1e3 * statistics.median(wall),
            "higher_is_better": True, "dtype": dtype_for(wl),
            "data": "synthetic", "config": {"workload": wl.name, "T": T, "experts": wl.n_experts,
                                            "top_k": wl.top_k, "cache_slots": args.cache_slots,
                                            "pool_gb": (wl.n_experts + wl.has_shared) * cfg.blob_bytes / 1e9},
            "cache": {"hit_rate": hits / max(1, hits + misses), "hits": hits, "misses": misses,
                      "h2d_bytes_per_token": nbytes / (K * T), "h2d_gbs": nbytes / total / 1e9},
            "how": "host clock per step: route, indices to the host, moe_cache_fetch (one DMA copy per missing "
                   "expert), moe_layer on the cached pool, synchronised; no L2 flush (the copies dominate)"}
    print(json.dumps(line), flush=True)


def int8_peak(path):
    """Dense int8 x int8 -> int32 GEMM throughput of the device (cuBLAS through
    torch._int_mm, 8192 x 8192 x 8192), CUDA events after warm-up: the
    denominator of the tensor-core path's utilisation."""
    import torch
    n = 8192
    a = torch.randint(-127, 128, (n, n), dtype=torch.int8, device="cuda")
    b = torch.randint(-127, 128, (n, n), dtype=torch.int8, device="cuda").t()
    for _ in range(5):
        torch._int_mm(a, b)
    torch.cuda.synchronize()
    ms = []
    for _ in range(20):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        torch._int_mm(a, b)
        e1.record()
        torch.cuda.synchronize()
        ms.append(e0.elapsed_time(e1))
    with Clocks(torch.cuda.current_device()) as clk:
        clk.wait_first()
        t0 = time.perf_counter()
        while time.perf_counter() - t0 < 3.0:  # sustained: seconds of back-to-back GEMMs
            torch._int_mm(a, b)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(50):
            torch._int_mm(a, b)
        e1.record()
        torch.cuda.synchronize()
        sus = e0.elapsed_time(e1) / 50
    ops = 2.0 * n ** 3
    rec = {"int8_tops_burst": ops / (statistics.median(ms) / 1e3) / 1e12,
           "int8_tops_sustained": ops / (sus / 1e3) / 1e12,
           "how": "torch._int_mm (cuBLAS) 8192^3 int8 -> int32, CUDA events; burst = median of 20 single GEMMs "
                  "after 5 warm-up, sustained = mean of 50 after 3 s of back-to-back GEMMs",
           "device": torch.cuda.get_device_name(), "clocks": clk.summary()}
    with open(path, "w") as fh:
        json.dump(rec, fh, indent=1)
    print(json.dumps(rec), flush=True)


def main(argv=None):
    args = parse(argv)
    if args.int8_peak:
        int8_peak(os.path.join(ROOT, "profiles", "int8_peak.json"))
        return
    import workloads as W
    wl = W.workload(args.workload)
    if args.n_experts:
        wl = wl.replace(n_experts=args.n_experts, name=f"{wl.name}_e{args.n_experts}")
    if args.tokens:
        wl = wl.replace(T=args.tokens, name=f"{wl.name}_T{args.tokens}")
    if args.topp:
        wl = wl.replace(topp=args.topp, name=f"{wl.name}_topp{args.topp:g}")
    if args.wbits and args.wbits != wl.wbits:
        tag, new = f"_int{wl.wbits}", f"_int{args.wbits}"
        name = wl.name.replace(tag, new) if tag in wl.name else wl.name + new
        wl = wl.replace(wbits=args.wbits, name=name)
    if args.impl == "reference":
        reference_arm(args, wl)
    elif args.cache_slots:
        cache_arm(args, wl)
    else:
        gpu_arm(args, wl)


if __name__ == "__main__":
    main()
