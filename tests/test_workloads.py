"""The seeded input generator: its published definition, its cross-device
determinism, and the fixed facts of the Colibri pages that the workload shapes
reproduce."""
import json
import os

import numpy as np
import pytest
import torch

import workloads as W

HERE = os.path.dirname(os.path.abspath(__file__))


def test_splitmix64_published_first_outputs():
    # SplitMix64 seeded with 0 (state advanced by GAMMA before mixing) starts
    # 0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F.
    got = [v & W.MASK64 for v in W.u64_stream(0, 0, 3).tolist()]
    assert got == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_counter_stream_slices_agree():
    k = W.stream_key(0, 7, 3, W.TAG_POOL)
    full = W.bytes_stream(k, 0, 4096)
    np.testing.assert_array_equal(W.bytes_stream(k, 1024, 1024).numpy(), full[1024:2048].numpy())
    ref = [W.mix64_int(k + (i + 1) * W.GAMMA) for i in range(4)]
    assert [v & W.MASK64 for v in W.u64_stream(k, 0, 4).tolist()] == ref


def test_pool_is_concatenation_of_expert_blobs():
    wl = W.workload(0)
    pool = W.pool_bytes(wl, 0, 0)
    for e in (0, 3, wl.n_experts):
        np.testing.assert_array_equal(pool[e * wl.blob_bytes:(e + 1) * wl.blob_bytes].numpy(),
                                      W.expert_blob(wl, 0, 0, e).numpy())
    sc = W.pool_scales(wl, 0, 0)
    np.testing.assert_array_equal(sc[5].numpy(), W.expert_scales(wl, 0, 0, 5).numpy())


def test_page_facts_bytes_per_expert_and_token():
    wl = W.workload(1)
    # ~19 MB per int4 expert (agentlenshq summary, "Memory split")
    assert wl.blob_bytes == 18_874_368
    assert abs(wl.blob_bytes + wl.scale_rows * 4 - 19e6) / 19e6 < 0.01
    # 75 MoE layers x top-8 x expert bytes ~ 11 GB per token (same page, perf section)
    per_token = 75 * 8 * (wl.blob_bytes + wl.scale_rows * 4)
    assert 10.5e9 < per_token < 11.8e9
    # routed experts of the whole model: 19,456 = 76 x 256 (remio.ai), ~370 GB
    assert 76 * 256 == 19_456 and 340e9 < 19_456 * wl.blob_bytes < 380e9
    # int2 experts are half the codes
    assert W.workload(4).blob_bytes == wl.blob_bytes // 2


def test_distributions():
    wl = W.workload(1)
    sc = W.pool_scales(wl, 0, 0).double().log()
    assert abs(sc.mean().item() + 4.0) < 0.01 and abs(sc.std().item() - 0.3) < 0.01
    wr = W.router_weight(wl, 0, 0)
    assert abs(wr.std().item() - 0.02) < 2e-4
    b = W.router_bias(wl, 0, 0)
    assert b.abs().max().item() <= 0.01
    x = W.tokens(wl, 0, 5).float()
    assert x.dtype == torch.float32 and abs(x.std().item() - 1) < 0.05
    blob = W.expert_blob(wl, 0, 0, 7).numpy()
    counts = np.bincount(blob & 0xF, minlength=16)
    assert counts.min() > 0.9 * blob.size / 16  # uniform int4 codes


def test_outlier_channels():
    wl = W.workload(3)
    ch = W.outlier_channels(wl, 0)
    assert ch.numel() == 61 and len(set(ch.tolist())) == 61
    x = W.tokens(wl, 0).float()
    ratio = x[:, ch].abs().mean() / x.abs().mean()
    assert ratio > 10


def test_zipf_beta_matches_calibration_file():
    with open(os.path.join(HERE, "golden", "zipf_beta.json")) as fh:
        rec = json.load(fh)
    assert W.workload(4).zipf_beta == rec["zipf_beta"] == W.ZIPF_BETA_SKEWED


def test_zipf_share_with_oracle_router():
    import oracle as O
    wl = W.workload(4)
    x_in = O.rmsnorm(W.tokens(wl, 0).float().numpy().astype(np.float64))
    idx, _ = O.route(x_in, W.router_weight(wl, 0, 0), W.router_bias(wl, 0, 0), wl.top_k)
    counts = np.sort(np.bincount(idx.reshape(-1), minlength=wl.n_experts))[::-1]
    assert abs(counts[:16].sum() / idx.size - 0.70) <= 0.02


@pytest.mark.gpu
def test_device_generation_matches_host():
    wl = W.workload(1)
    k = W.stream_key(0, 1, 2, 3)
    a = W.bytes_stream(k, 8 * 12345, 1 << 20, "cuda").cpu()
    b = W.bytes_stream(k, 8 * 12345, 1 << 20, "cpu")
    assert torch.equal(a, b)
    out = torch.empty(wl.blob_bytes * 2, dtype=torch.uint8, device="cuda")
    W.fill_bytes_(out, W._key(wl, 0, 0, W.TAG_POOL), byte_start=5 * wl.blob_bytes)
    assert torch.equal(out[wl.blob_bytes:].cpu(), W.expert_blob(wl, 0, 0, 6))
