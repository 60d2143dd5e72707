"""CPU oracle of the routed-expert MoE layer -- TEST INFRASTRUCTURE ONLY.

Only tests/, ``__graft_entry__.smoke()`` and bench.py's cpu_baseline and
reference legs may import this package.  The product (expert_ffn_router_b200)
never imports it, and it never imports the product: the two share no code; the
seeded inputs come from the separate ``workloads`` module.

The arithmetic lives in oracle.c (plain C, see its header for what each step
computes and which passage of the Colibri pages it follows).  This file is
ctypes marshalling plus the host-side orchestration of multi-layer runs
(parameter-free RMSNorm + residual between layers) and of regenerating only the
experts a token actually selects.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

from . import build as _build

_lib = None

_P = ctypes.c_void_p
_I = ctypes.c_int
_D = ctypes.c_double
_I64 = ctypes.c_int64


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.oracle_num_threads.restype = _I
        L.oracle_set_num_threads.argtypes = [_I]
        L.oracle_unpack.argtypes = [_I, _P, _I64, _P]
        L.oracle_pack.argtypes = [_I, _P, _I64, _P]
        L.oracle_quantize.argtypes = [_P, _I, _I, _P, _P]
        L.oracle_route.argtypes = [_P, _I, _I, _I, _I, _P, _P, _D, _P, _P, _P, _P, _P]
        L.oracle_route_p.argtypes = [_P, _I, _I, _I, _I, _P, _P, _D, ctypes.c_float, _P, _P, _P, _P, _P]
        L.oracle_down.argtypes = [_I, _I, _I, _P, _P, _P, _P, _I, _P, _P]
        L.oracle_expert.argtypes = [_I, _I, _I, _P, _P, _P, _P, _I, _P, _P, _P, _P, _P, _P]
        L.oracle_layer.argtypes = [_I, _I, _I, _I, _I, _I, _D, _P, _P, _P, _P, _P, _I, _P, _P, _P,
                                   _P, _P]
        L.oracle_layer_p.argtypes = [_I, _I, _I, _I, _I, _I, _D, ctypes.c_float, _P, _P, _P, _P, _P, _I, _P,
                                     _P, _P, _P, _P]
        L.oracle_rmsnorm.argtypes = [_P, _I, _I, _D, _P]
        for fn in ("oracle_unpack", "oracle_pack", "oracle_quantize", "oracle_route", "oracle_route_p",
                   "oracle_down", "oracle_expert", "oracle_layer", "oracle_layer_p", "oracle_rmsnorm"):
            getattr(L, fn).restype = _I
        _lib = L
    return _lib


def _ptr(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"{what} failed with code {rc}")


def _np(a, dtype) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().cpu()
        if str(a.dtype) == "torch.bfloat16":
            a = a.float()
        a = a.numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=dtype))


def num_threads() -> int:
    return lib().oracle_num_threads()


def set_num_threads(n: int):
    lib().oracle_set_num_threads(n)


def unpack(wbits: int, packed, n: int) -> np.ndarray:
    src = _np(packed, np.uint8)
    out = np.empty(n, np.int8)
    _check(lib().oracle_unpack(wbits, _ptr(src), n, _ptr(out)), "oracle_unpack")
    return out


def pack(wbits: int, codes) -> np.ndarray:
    src = _np(codes, np.int8)
    out = np.empty(src.size * wbits // 8, np.uint8)
    _check(lib().oracle_pack(wbits, _ptr(src), src.size, _ptr(out)), "oracle_pack")
    return out


def quantize(x) -> Tuple[np.ndarray, np.ndarray]:
    x = _np(x, np.float32)
    T, d = x.shape
    q = np.empty((T, d), np.int8)
    s = np.empty(T, np.float32)
    _check(lib().oracle_quantize(_ptr(x), T, d, _ptr(q), _ptr(s)), "oracle_quantize")
    return q, s


def route(x, w_router, bias, k: int, routed_scale: float = 2.5, want_scores: bool = False, topp: float = 0.0):
    """Returns idx int32 [T][k], w float64 [T][k] (and logits, s, sel fp32 [T][E]).
    topp in (0, 1): TOPP truncation (oracle.c, a1'): dropped slots idx -1, w 0."""
    x = _np(x, np.float32)
    wr = _np(w_router, np.float32)
    b = _np(bias, np.float32)
    T, d = x.shape
    E = wr.shape[0]
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    lg = np.empty((T, E), np.float32) if want_scores else None
    s = np.empty((T, E), np.float32) if want_scores else None
    sel = np.empty((T, E), np.float32) if want_scores else None
    _check(lib().oracle_route_p(_ptr(x), T, d, E, k, _ptr(wr), _ptr(b), routed_scale, topp, _ptr(idx),
                                _ptr(w), _ptr(lg), _ptr(s), _ptr(sel)), "oracle_route_p")
    if want_scores:
        return idx, w, lg, s, sel
    return idx, w


def expert(d: int, f: int, wbits: int, blob, scales, xq, sx) -> Dict[str, np.ndarray]:
    """One expert over T tokens; returns every intermediate."""
    blob = _np(blob, np.uint8)
    sc = _np(scales, np.float32)
    xq = _np(xq, np.int8)
    sx = _np(sx, np.float32)
    T = xq.shape[0]
    r = dict(acc_gu=np.empty((T, 2 * f), np.int32), h=np.empty((T, f), np.float32),
             hq=np.empty((T, f), np.int8), sh=np.empty(T, np.float32),
             acc_d=np.empty((T, d), np.int32), y=np.empty((T, d), np.float64))
    _check(lib().oracle_expert(d, f, wbits, _ptr(blob), _ptr(sc), _ptr(xq), _ptr(sx), T,
                               _ptr(r["acc_gu"]), _ptr(r["h"]), _ptr(r["hq"]), _ptr(r["sh"]),
                               _ptr(r["acc_d"]), _ptr(r["y"])), "oracle_expert")
    return r


def down(d: int, f: int, wbits: int, blob, scales, hq, sh) -> Dict[str, np.ndarray]:
    blob = _np(blob, np.uint8)
    sc = _np(scales, np.float32)
    hq = _np(hq, np.int8)
    sh = _np(sh, np.float32)
    T = hq.shape[0]
    r = dict(acc_d=np.empty((T, d), np.int32), y=np.empty((T, d), np.float64))
    _check(lib().oracle_down(d, f, wbits, _ptr(blob), _ptr(sc), _ptr(hq), _ptr(sh), T,
                             _ptr(r["acc_d"]), _ptr(r["y"])), "oracle_down")
    return r


def layer(d: int, f: int, E: int, k: int, has_shared: int, wbits: int, routed_scale: float,
          blobs: Sequence[Optional[np.ndarray]], scales: Sequence[Optional[np.ndarray]], w_router,
          bias, x, topp: float = 0.0) -> Dict[str, np.ndarray]:
    """Full layer on x fp32 [T][d].  blobs/scales: per-expert arrays (shared last);
    entries may be None for experts no token selects."""
    x = _np(x, np.float32)
    wr = _np(w_router, np.float32)
    b = _np(bias, np.float32)
    T = x.shape[0]
    n = E + has_shared
    assert len(blobs) == n and len(scales) == n
    keep = [(_np(bb, np.uint8) if bb is not None else None) for bb in blobs]
    keep_s = [(_np(ss, np.float32) if ss is not None else None) for ss in scales]
    bt = (ctypes.c_void_p * n)(*[_ptr(a) for a in keep])
    st = (ctypes.c_void_p * n)(*[_ptr(a) for a in keep_s])
    out = np.empty((T, d), np.float64)
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    xq = np.empty((T, d), np.int8)
    sx = np.empty(T, np.float32)
    _check(lib().oracle_layer_p(d, f, E, k, has_shared, wbits, routed_scale, topp, ctypes.cast(bt, _P),
                                ctypes.cast(st, _P), _ptr(wr), _ptr(b), _ptr(x), T, _ptr(out),
                                _ptr(idx), _ptr(w), _ptr(xq), _ptr(sx)), "oracle_layer_p")
    return dict(out=out, idx=idx, w=w, xq=xq, sx=sx)


def rmsnorm(x64, eps: float = 1e-6) -> np.ndarray:
    x = _np(x64, np.float64)
    T, d = x.shape
    y = np.empty((T, d), np.float32)
    _check(lib().oracle_rmsnorm(_ptr(x), T, d, eps, _ptr(y)), "oracle_rmsnorm")
    return y


# ---------------------------------------------------------------------------
# Orchestration over the seeded workloads (pulls inputs from ``workloads``).
# ---------------------------------------------------------------------------
def workload_layer(wl, seed: int, layer_idx: int, x_in, L=None, blob_cache=None):
    """Run one layer of a seeded workload on x_in fp32 [T][d], regenerating only
    the expert blobs the oracle's own routing selects."""
    import workloads as W
    if L is None:
        L = W.layer(wl, seed, layer_idx)
    x_in = _np(x_in, np.float32)
    topp = getattr(wl, "topp", 0.0)
    idx, _ = route(x_in, L.w_router, L.bias, wl.top_k, wl.routed_scale, topp=topp)
    need = sorted((set(idx.reshape(-1).tolist()) - {-1}) | ({wl.n_experts} if wl.has_shared else set()))
    blobs: List[Optional[np.ndarray]] = [None] * wl.n_blobs
    scales: List[Optional[np.ndarray]] = [None] * wl.n_blobs
    sc_all = L.scales.numpy()
    for e in need:
        key = (layer_idx, e)
        if blob_cache is not None and key in blob_cache:
            blobs[e] = blob_cache[key]
        else:
            blobs[e] = W.expert_blob(wl, seed, layer_idx, e).numpy()
            if blob_cache is not None:
                blob_cache[key] = blobs[e]
        scales[e] = np.ascontiguousarray(sc_all[e])
    return layer(wl.d, wl.f, wl.n_experts, wl.top_k, wl.has_shared, wl.wbits, wl.routed_scale,
                 blobs, scales, L.w_router, L.bias, x_in, topp=topp)


def workload_stack(wl, seed: int, x0, n_layers: Optional[int] = None, eps: float = 1e-6,
                   blob_cache=None) -> Dict[str, list]:
    """Stacked layers: x_in = RMSNorm(x); x <- x + layer(x_in).  Residual in fp64.
    Returns the final residual and each layer's idx and x_in."""
    n_layers = wl.n_layers if n_layers is None else n_layers
    x = _np(x0, np.float32).astype(np.float64)
    idxs, xins, outs = [], [], []
    for l in range(n_layers):
        x_in = rmsnorm(x, eps)
        r = workload_layer(wl, seed, l, x_in, blob_cache=blob_cache)
        x = x + r["out"]
        idxs.append(r["idx"])
        xins.append(x_in)
        outs.append(r["out"])
    return dict(x=x, idx=idxs, x_in=xins, out=outs)
