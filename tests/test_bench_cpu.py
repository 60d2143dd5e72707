"""bench.py's host logic without a GPU: the reference arm's JSON line, the
rank handling of the multi-GPU launch (two gloo ranks on the CPU), and the
per-rank token streams."""
import argparse
import contextlib
import datetime
import io
import json
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
import workloads as W  # noqa: E402


def args_for(workload, steps=2, warmup=3, gpus=1):
    return argparse.Namespace(steps=steps, warmup=warmup, gpus=gpus, workload=workload, layers=0)


def run_reference(workload, monkeypatch, rank="0"):
    monkeypatch.setenv("RANK", rank)
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.reference_arm(args_for(workload), W.workload(workload))
    return buf.getvalue().strip()


def test_reference_arm_line(monkeypatch):
    out = run_reference(0, monkeypatch)
    line = json.loads(out)
    wl = W.workload(0)
    assert line["impl"] == "reference"
    assert line["metric"] == bench.metric_for(wl, 0) and line["unit"] == "tokens/s"
    assert line["value"] > 0 and line["ms_per_step"] > 0
    assert line["steps"] == 2 and line["warmup"] == 3 and line["n_gpus"] == 1
    assert line["higher_is_better"] is True and line["scaling"] == "weak" and line["vs_baseline"] is None
    assert line["dtype"] == "i8*i4->i32" and line["data"] == "synthetic"
    assert line["config"]["workload"] == wl.name
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1 and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_print_nothing(monkeypatch):
    assert run_reference(0, monkeypatch, rank="1") == ""


def test_labels():
    assert bench.metric_for(W.workload(1), 1) == bench.METRIC
    assert bench.metric_for(W.workload(3), 3) != bench.METRIC
    assert bench.dtype_for(W.workload(1)) == "i8*i4->i32"
    assert bench.dtype_for(W.workload(4)) == "i8*i2->i32"
    # a modified headline workload (int8 codes, truncation, more tokens) is
    # a labelled variant, not the headline metric
    int8 = W.workload(1).replace(wbits=8, name=W.workload(1).name + "_int8")
    assert bench.dtype_for(int8) == "i8*i8->i32"
    assert bench.metric_for(int8, 1) != bench.METRIC and int8.name in bench.metric_for(int8, 1)
    topp = W.workload(1).replace(topp=0.7, name=W.workload(1).name + "_topp0.7")
    assert bench.metric_for(topp, 1) != bench.METRIC


def test_variant_options_name_the_workload(monkeypatch):
    seen = {}
    monkeypatch.setattr(bench, "gpu_arm", lambda args, wl: seen.update(wl=wl))
    bench.main(["--wbits", "8", "--tokens", "8", "--topp", "0.7"])
    wl = seen["wl"]
    assert (wl.wbits, wl.T, wl.topp) == (8, 8, 0.7)
    assert wl.name == "decode_T1_d6144_f2048_e256_k8_int8_T8_topp0.7"
    bench.main(["--wbits", "4"])  # the workload's own width: unchanged
    assert seen["wl"] == W.workload(1)


def test_rank_token_streams():
    assert bench.rank_token_sets(0, 3) == [0, 1, 2]  # rank 0 is the single-GPU stream
    r0, r1 = set(bench.rank_token_sets(0, 100)), set(bench.rank_token_sets(1, 100))
    assert not r0 & r1
    wl = W.workload(1)
    assert not torch.equal(W.tokens(wl, 0, bench.rank_token_sets(0, 1)[0]),
                           W.tokens(wl, 0, bench.rank_token_sets(1, 1)[0]))


def test_whole_job_rate():
    # two ranks, 10 steps of 1 token, the slower rank took 20 ms in total
    assert bench.whole_job_rate(2, 10, 1, 20.0) == pytest.approx(1000.0)
    assert bench.max_over_ranks(3.5, 1) == 3.5


def _rank_main(rank, world, port, outdir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        local = [12.5, 30.25][rank]  # each rank's own total time
        m = bench.max_over_ranks(local, world, dist, "cpu")
        e2e = bench.max_over_ranks(local * 2, world, dist, "cpu")  # the same collectives, same order
        with open(os.path.join(outdir, f"r{rank}.json"), "w") as fh:
            json.dump({"max": m, "e2e": e2e, "rate": bench.whole_job_rate(world, 10, 1, m)}, fh)
    finally:
        dist.destroy_process_group()


def test_max_over_two_gloo_ranks(tmp_path):
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    mp.spawn(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True)
    res = [json.load(open(tmp_path / f"r{r}.json")) for r in range(2)]
    for r in res:
        assert r["max"] == 30.25 and r["e2e"] == 60.5
        assert r["rate"] == pytest.approx(2 * 10 * 1 / 0.03025)
