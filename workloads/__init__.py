"""Seeded synthetic inputs for the routed-expert MoE layer.

This module only draws numbers; it holds none of the layer's arithmetic (no
routing, no quantisation, no dot products).  Both the CPU oracle and the CUDA
path take their inputs from here, so the two sides see identical bytes.

Generator: SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom
number generators", OOPSLA 2014), used counter-style: draw ``i`` of stream
``key`` is ``mix64(key + (i + 1) * GAMMA)`` modulo 2**64, so any slice of any
stream can be regenerated on its own (one expert's blob on the host, the whole
pool on the device).  Integer draws (the packed weight codes) are pure 64-bit
integer arithmetic and come out bit-identical on CPU and CUDA.  Float draws
(scales, router, bias, activations) are made on the host in float64 and then
rounded (to float32, and to bfloat16 by round-to-nearest-even from float32).

Workload shapes follow the Colibri pages: the tiny ``glm_tiny`` fixture
(hidden 128, 8 experts per layer, top-2; takumi3488 article, coli info log) and
the real GLM-5.2 MoE layer (hidden 6144, 256 experts per layer, top-8; same
article, coli info log of the int4 model), with ~19 MB int4 experts (agentlenshq
summary, "Memory split").  The intermediate width f = 2048 is the value at
which 3*d*f/2 bytes of int4 codes give the ~19 MB per expert those pages state.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

MASK64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15
MIX1 = 0xBF58476D1CE4E5B9
MIX2 = 0x94D049BB133111EB

# stream tags
TAG_POOL, TAG_SCALES, TAG_ROUTER, TAG_BIAS, TAG_X, TAG_OUTLIER, TAG_ZIPF = 1, 2, 3, 4, 5, 6, 7


def _signed(c: int) -> int:
    return c - (1 << 64) if c >= (1 << 63) else c


_GAMMA_S, _MIX1_S, _MIX2_S = _signed(GAMMA), _signed(MIX1), _signed(MIX2)


def mix64_int(z: int) -> int:
    """SplitMix64 finaliser on a Python int (mod 2**64)."""
    z &= MASK64
    z = ((z ^ (z >> 30)) * MIX1) & MASK64
    z = ((z ^ (z >> 27)) * MIX2) & MASK64
    return z ^ (z >> 31)


def stream_key(seed: int, *labels: int) -> int:
    """Key of one named stream: the seed folded with each label through mix64."""
    k = mix64_int(seed + GAMMA)
    for lab in labels:
        k = mix64_int(k ^ ((lab + GAMMA) & MASK64))
    return k


def _lsr(x: torch.Tensor, s: int) -> torch.Tensor:
    """Logical right shift of int64 lanes (torch's >> is arithmetic)."""
    return (x >> s) & ((1 << (64 - s)) - 1)


def u64_stream(key: int, start: int, count: int, device="cpu") -> torch.Tensor:
    """Draws ``start .. start+count-1`` of stream ``key`` as int64 lanes holding
    the 64-bit pattern (two's complement wrap on both CPU and CUDA)."""
    i = torch.arange(start + 1, start + 1 + count, dtype=torch.int64, device=device)
    z = i * _GAMMA_S + _signed(key & MASK64)
    z = (z ^ _lsr(z, 30)) * _MIX1_S
    z = (z ^ _lsr(z, 27)) * _MIX2_S
    return z ^ _lsr(z, 31)


def bytes_stream(key: int, byte_start: int, nbytes: int, device="cpu") -> torch.Tensor:
    """Bytes of stream ``key`` (draw i gives bytes 8i..8i+7, little-endian) as uint8."""
    assert byte_start % 8 == 0 and nbytes % 8 == 0
    return u64_stream(key, byte_start // 8, nbytes // 8, device).view(torch.uint8)


def fill_bytes_(out: torch.Tensor, key: int, byte_start: int = 0, chunk: int = 1 << 27) -> torch.Tensor:
    """Fill a flat uint8 tensor (any device) with stream bytes, in bounded chunks."""
    flat = out.view(-1)
    n = flat.numel()
    assert n % 8 == 0
    for off in range(0, n, chunk):
        m = min(chunk, n - off)
        flat[off:off + m] = bytes_stream(key, byte_start + off, m, out.device)
    return out


def _unit(u: torch.Tensor) -> torch.Tensor:
    """Top 53 bits of each draw as float64 in [0, 1)."""
    return _lsr(u, 11).to(torch.float64) * (2.0 ** -53)


def uniform01(key: int, start: int, count: int) -> torch.Tensor:
    return _unit(u64_stream(key, start, count))


def normal(key: int, start: int, count: int) -> torch.Tensor:
    """Standard normals in float64 (Box-Muller, cosine branch): element i uses
    draws 2i and 2i+1 of the stream."""
    u = _unit(u64_stream(key, 2 * start, 2 * count)).view(count, 2)
    r = torch.sqrt(-2.0 * torch.log1p(-u[:, 0]))  # 1-u in (0, 1]
    return r * torch.cos(2.0 * math.pi * u[:, 1])


def permutation(key: int, n: int) -> torch.Tensor:
    """Seeded permutation of 0..n-1: stable argsort of n stream draws (top 62 bits)."""
    return torch.argsort(_lsr(u64_stream(key, 0, n), 2), stable=True)


def to_bf16(x64: torch.Tensor) -> torch.Tensor:
    return x64.to(torch.float32).to(torch.bfloat16)


# ---------------------------------------------------------------------------
# Workload configurations
# ---------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    d: int
    f: int
    n_experts: int
    top_k: int
    has_shared: int
    wbits: int
    T: int
    n_layers: int
    x_dtype: str          # "f32" or "bf16"
    n_token_sets: int = 1  # distinct seeded token batches (decode draws one per step)
    outlier_frac: float = 0.0
    outlier_mult: float = 1.0
    zipf_s: float = 0.0
    zipf_beta: float = 0.0
    routed_scale: float = 2.5
    bias_halfwidth: float = 0.01
    residual: bool = False
    topp: float = 0.0     # TOPK/TOPP truncation threshold of the router (0 = off)

    @property
    def blob_bytes(self) -> int:
        return 3 * self.d * self.f * self.wbits // 8

    @property
    def n_blobs(self) -> int:
        return self.n_experts + self.has_shared

    @property
    def pool_bytes(self) -> int:
        return self.n_blobs * self.blob_bytes

    @property
    def scale_rows(self) -> int:
        return 2 * self.f + self.d

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The Zipf amplitude beta of the skewed-routing workload: the value at which, on
# layer 0's draws, the 16 most-assigned experts take 70% (+-2%) of the 512
# assignments.  Written by tests/golden/calibrate_zipf_beta.py, which calls only
# the CPU oracle; tests/test_workloads.py re-checks the share with the oracle.
ZIPF_BETA_SKEWED = 2.379300594329834

WORKLOADS = {
    0: Workload("tiny_d128_f64_e8_k2_T32", 128, 64, 8, 2, 1, 4, 32, 1, "f32"),
    1: Workload("decode_T1_d6144_f2048_e256_k8_int4", 6144, 2048, 256, 8, 1, 4, 1, 1, "bf16",
                n_token_sets=100),
    2: Workload("mtp_verify_T4_8layers_int4", 6144, 2048, 256, 8, 1, 4, 4, 8, "bf16", residual=True),
    3: Workload("prefill_T512_int4_outliers", 6144, 2048, 256, 8, 1, 4, 512, 1, "bf16",
                outlier_frac=0.01, outlier_mult=20.0),
    4: Workload("skewed_T64_24layers_int2_zipf", 6144, 2048, 256, 8, 1, 2, 64, 24, "bf16",
                zipf_s=1.1, zipf_beta=ZIPF_BETA_SKEWED, residual=True),
}


def workload(i: int) -> Workload:
    return WORKLOADS[i]


# ---------------------------------------------------------------------------
# Per-layer tensors.  Every draw is keyed on (seed, workload id, layer, tag).
# ---------------------------------------------------------------------------
def _key(wl: Workload, seed: int, layer: int, tag: int) -> int:
    return stream_key(seed, _wid(wl), layer, tag)


def _wid(wl: Workload) -> int:
    # workload identity for stream keys: the dims that change the bytes
    return (wl.d * 1000003 + wl.f * 10007 + wl.n_experts * 101 + wl.wbits) & 0xFFFFFFFF


def expert_blob(wl: Workload, seed: int, layer: int, e: int, device="cpu") -> torch.Tensor:
    """Packed code bytes of expert ``e`` (``e == n_experts`` is the shared expert):
    ``blob_bytes`` uint8 laid out [gate f x d | up f x d | down d x f]."""
    B = wl.blob_bytes
    return bytes_stream(_key(wl, seed, layer, TAG_POOL), e * B, B, device)


def pool_bytes(wl: Workload, seed: int, layer: int, device="cpu", out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """All ``n_blobs`` blobs of one layer, contiguous (expert e at offset e*blob_bytes)."""
    if out is None:
        out = torch.empty(wl.pool_bytes, dtype=torch.uint8, device=device)
    return fill_bytes_(out, _key(wl, seed, layer, TAG_POOL))


def expert_scales(wl: Workload, seed: int, layer: int, e: int) -> torch.Tensor:
    """fp32 per-output-row scales of expert ``e``: [gate f | up f | down d],
    lognormal(mu=-4, sigma=0.3)."""
    R = wl.scale_rows
    z = normal(_key(wl, seed, layer, TAG_SCALES), e * R, R)
    return torch.exp(-4.0 + 0.3 * z).to(torch.float32)


def pool_scales(wl: Workload, seed: int, layer: int) -> torch.Tensor:
    R = wl.scale_rows
    z = normal(_key(wl, seed, layer, TAG_SCALES), 0, wl.n_blobs * R)
    return torch.exp(-4.0 + 0.3 * z).to(torch.float32).view(wl.n_blobs, R)


def router_weight(wl: Workload, seed: int, layer: int) -> torch.Tensor:
    """fp32 [E][d], N(0, 0.02^2)."""
    z = normal(_key(wl, seed, layer, TAG_ROUTER), 0, wl.n_experts * wl.d)
    return (0.02 * z).to(torch.float32).view(wl.n_experts, wl.d)


def zipf_ranks(wl: Workload, seed: int, layer: int) -> torch.Tensor:
    """rank[e] of each expert in the Zipf bias (0 = most favoured)."""
    perm = permutation(_key(wl, seed, layer, TAG_ZIPF), wl.n_experts)
    rank = torch.empty_like(perm)
    rank[perm] = torch.arange(wl.n_experts)
    return rank


def router_bias(wl: Workload, seed: int, layer: int, zipf_beta: Optional[float] = None) -> torch.Tensor:
    """fp32 [E]: uniform(-h, h), plus beta*(rank+1)^-s for the Zipf workload."""
    u = uniform01(_key(wl, seed, layer, TAG_BIAS), 0, wl.n_experts)
    b = -wl.bias_halfwidth + 2.0 * wl.bias_halfwidth * u
    beta = wl.zipf_beta if zipf_beta is None else zipf_beta
    if wl.zipf_s > 0.0 and beta != 0.0:
        rank = zipf_ranks(wl, seed, layer).to(torch.float64)
        b = b + beta * torch.pow(rank + 1.0, -wl.zipf_s)
    return b.to(torch.float32)


def outlier_channels(wl: Workload, seed: int) -> torch.Tensor:
    n = int(math.floor(wl.outlier_frac * wl.d))
    return torch.sort(permutation(stream_key(seed, _wid(wl), 0, TAG_OUTLIER), wl.d)[:n]).values


def tokens(wl: Workload, seed: int, token_set: int = 0, T: Optional[int] = None) -> torch.Tensor:
    """Activations [T][d]: N(0,1), outlier channels scaled before rounding;
    float32 for the tiny workload, bfloat16 otherwise."""
    T = wl.T if T is None else T
    z = normal(stream_key(seed, _wid(wl), token_set, TAG_X), 0, T * wl.d).view(T, wl.d)
    if wl.outlier_frac > 0.0:
        z[:, outlier_channels(wl, seed)] *= wl.outlier_mult
    if wl.x_dtype == "f32":
        return z.to(torch.float32)
    return to_bf16(z)


@dataclasses.dataclass
class Layer:
    """One layer's inputs on the host (the pool bytes are filled on demand)."""
    wl: Workload
    seed: int
    layer: int
    scales: torch.Tensor    # fp32 [n_blobs][2f+d]
    w_router: torch.Tensor  # fp32 [E][d]
    bias: torch.Tensor      # fp32 [E]


def layer(wl: Workload, seed: int, layer_idx: int) -> Layer:
    return Layer(wl, seed, layer_idx, pool_scales(wl, seed, layer_idx),
                 router_weight(wl, seed, layer_idx), router_bias(wl, seed, layer_idx))


@dataclasses.dataclass
class DeviceLayer:
    """One layer's inputs resident on a device (pool bytes generated there)."""
    pool_w: torch.Tensor    # uint8 [n_blobs * blob_bytes]
    pool_s: torch.Tensor    # fp32 [n_blobs][2f+d]
    w_router: torch.Tensor  # fp32 [E][d]
    bias: torch.Tensor      # fp32 [E]


def device_layer(wl: Workload, seed: int, layer_idx: int, device="cuda", host: Optional[Layer] = None) -> DeviceLayer:
    L = host if host is not None else layer(wl, seed, layer_idx)
    w = pool_bytes(wl, seed, layer_idx, device=device)
    return DeviceLayer(w, L.scales.to(device), L.w_router.to(device), L.bias.to(device))
