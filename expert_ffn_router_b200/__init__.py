"""Python binding of libmoe, the sm_100a routed-expert MoE layer library.

Argument marshalling only: every function below checks that its torch tensors
have the dtype and shape the C ABI expects, passes their device pointers and
the current CUDA stream to the function of the same name in libmoe.so
(include/moe.h), and raises ``MoeError`` on a non-zero status.  Every step of
the layer runs in the library's kernels; there is no fallback: if libmoe.so
is missing or fails to load, importing this package raises.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# MOE_LIBRARY=bounds loads the bounds-checked build (every index the kernels
# read from data range-checked into the status word), for tests
LIB_PATH = os.path.join(_PKG, "libmoe_bounds.so" if os.environ.get("MOE_LIBRARY") == "bounds" else "libmoe.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "moe.h")

MOE_OK, MOE_EINVAL, MOE_EALIGN, MOE_ENOSPACE, MOE_ECUDA, MOE_ETIMEOUT, MOE_EDEVICE = 0, -1, -2, -3, -4, -5, -6
MOE_IO_X_HOST, MOE_IO_OUT_HOST = 1, 2  # moe_layer_opts.io_host bits
MOE_F32, MOE_BF16 = 0, 1
MOE_PATH_AUTO, MOE_PATH_MULTI, MOE_PATH_DECODE, MOE_PATH_TC = 0, 1, 2, 3


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        super().__init__(f"{where}: status {status}: {detail}")
        self.status = status


class MoeConfig(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("f", ctypes.c_int32), ("n_experts", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("has_shared", ctypes.c_int32), ("wbits", ctypes.c_int32),
                ("routed_scale", ctypes.c_float), ("tc_min_tokens", ctypes.c_int32), ("topp", ctypes.c_float)]

    @property
    def blob_bytes(self) -> int:
        return 3 * self.d * self.f * self.wbits // 8

    @property
    def n_blobs(self) -> int:
        return self.n_experts + self.has_shared

    @property
    def scale_rows(self) -> int:
        return 2 * self.f + self.d


class MoeLayerOpts(ctypes.Structure):
    _fields_ = [("events", ctypes.c_void_p * 4), ("path", ctypes.c_int32), ("n_launches", ctypes.c_int32),
                ("trace", ctypes.c_void_p), ("path_ran", ctypes.c_int32),
                ("wait_limit_us", ctypes.c_int32), ("test_skip_h", ctypes.c_int32), ("io_host", ctypes.c_int32)]


class MoePool(ctypes.Structure):
    _fields_ = [("w", ctypes.c_void_p), ("s", ctypes.c_void_p), ("slot_of", ctypes.c_void_p),
                ("n_slots", ctypes.c_int32)]


class MoeCache(ctypes.Structure):
    _fields_ = [("host_w", ctypes.c_void_p), ("slots", ctypes.c_void_p), ("slot_of", ctypes.c_void_p),
                ("state", ctypes.c_void_p), ("n_slots", ctypes.c_int32)]


class MoeCacheStats(ctypes.Structure):
    _fields_ = [("hits", ctypes.c_int64), ("misses", ctypes.c_int64), ("bytes", ctypes.c_int64)]


def config(d: int, f: int, n_experts: int, top_k: int, has_shared: int = 1, wbits: int = 4,
           routed_scale: float = 2.5, tc_min_tokens: int = 0, topp: float = 0.0) -> MoeConfig:
    return MoeConfig(d, f, n_experts, top_k, has_shared, wbits, routed_scale, tc_min_tokens, topp)


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python expert_ffn_router_b200/build.py`")
    L = ctypes.CDLL(LIB_PATH)
    P, I32, SZ, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t, ctypes.c_float
    C = ctypes.POINTER(MoeConfig)
    PL = ctypes.POINTER(MoePool)
    sig = {
        "moe_workspace_bytes": (SZ, [C, I32]),
        "moe_workspace_init": (I32, [P, SZ, P]),
        "moe_quantize": (I32, [C, P, I32, I32, P, P, P]),
        "moe_route": (I32, [C, P, I32, I32, P, P, P, P, P, SZ, P]),
        "moe_route_static": (I32, [C, P, I32, I32, P, P, P, P, P]),
        "moe_expert_ffn": (I32, [C, PL, I32, P, P, I32, P, P, P, P, P, P, SZ, P]),
        "moe_expert_down": (I32, [C, PL, I32, P, P, I32, P, P, P, SZ, P]),
        "moe_layer": (I32, [C, PL, P, P, P, I32, I32, P, I32, P, P, P, SZ, P]),
        "moe_layer_ex": (I32, [C, PL, P, P, P, I32, I32, P, I32, P, P, P, SZ, P, ctypes.POINTER(MoeLayerOpts)]),
        "moe_rmsnorm": (I32, [P, I32, I32, I32, F, P, P, P]),
        "moe_poll_status": (I32, [P, ctypes.POINTER(I32), P]),
        "moe_cache_state_bytes": (SZ, [C, I32]),
        "moe_cache_init": (I32, [C, ctypes.POINTER(MoeCache), P]),
        "moe_cache_fetch": (I32, [C, ctypes.POINTER(MoeCache), P, I32, P, ctypes.POINTER(MoeCacheStats)]),
        "moe_status_string": (ctypes.c_char_p, [I32]),
        "moe_last_error": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    return L


lib = _load()


def declared_symbols() -> list:
    """Names of the entry points include/moe.h declares."""
    with open(HEADER) as fh:
        return re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", fh.read())


def _check(st: int, where: str):
    if st != MOE_OK:
        raise MoeError(st, where, lib.moe_last_error().decode())


def _stream(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ptr(t: Optional[torch.Tensor], dtype=None, numel: Optional[int] = None, name: str = "",
         host: bool = False) -> Optional[int]:
    if t is None:
        return None
    if host:
        if t.is_cuda or not t.is_pinned():
            raise ValueError(f"{name}: expected a pinned host tensor")
    elif not t.is_cuda:
        raise ValueError(f"{name}: expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name}: expected {dtype}, got {t.dtype}")
    if numel is not None and t.numel() != numel:
        raise ValueError(f"{name}: expected {numel} elements, got {t.numel()}")
    return t.data_ptr()


def _xdtype(x: torch.Tensor) -> int:
    if x.dtype == torch.float32:
        return MOE_F32
    if x.dtype == torch.bfloat16:
        return MOE_BF16
    raise ValueError(f"x must be float32 or bfloat16, got {x.dtype}")


def make_pool(w: torch.Tensor, s: torch.Tensor, slot_of: Optional[torch.Tensor] = None,
              n_slots: int = 0) -> MoePool:
    """The C struct over device tensors; it keeps references to them, so their
    memory stays allocated for as long as the struct is in use.  With
    ``slot_of`` (an HBM expert cache's slot table) ``w`` holds ``n_slots``
    blobs."""
    pool = MoePool(_ptr(w, torch.uint8, name="pool.w"), _ptr(s, torch.float32, name="pool.s"),
                   _ptr(slot_of, torch.int32, name="pool.slot_of"), n_slots if slot_of is not None else 0)
    pool._tensors = (w, s, slot_of)
    return pool


class ExpertCache:
    """An HBM expert cache over one layer's pool in pinned host memory
    (moe_cache_init / moe_cache_fetch): ``n_slots`` device blobs, the slot
    table and the host book-keeping, all owned here.  ``pool`` is the
    moe_pool over the slots to pass to moe_layer after ``fetch``."""

    def __init__(self, cfg: MoeConfig, host_w: torch.Tensor, scales: torch.Tensor, n_slots: int, device="cuda",
                 stream=None):
        if host_w.is_cuda or not host_w.is_pinned():
            raise ValueError("host_w: expected a pinned host tensor")
        self.cfg = cfg
        B = cfg.blob_bytes
        self.host_w = host_w
        self.slots = torch.empty(n_slots * B, dtype=torch.uint8, device=device)
        self.slot_of = torch.empty(cfg.n_experts + cfg.has_shared, dtype=torch.int32, device=device)
        nb = lib.moe_cache_state_bytes(ctypes.byref(cfg), n_slots)
        if nb == 0:
            raise MoeError(MOE_EINVAL, "moe_cache_state_bytes", lib.moe_last_error().decode())
        self.state = (ctypes.c_uint64 * ((nb + 7) // 8))()
        self.c = MoeCache(host_w.data_ptr(), self.slots.data_ptr(), self.slot_of.data_ptr(),
                          ctypes.addressof(self.state), n_slots)
        self.pool = make_pool(self.slots, scales, self.slot_of, n_slots)
        _check(lib.moe_cache_init(ctypes.byref(cfg), ctypes.byref(self.c), _stream(stream)), "moe_cache_init")

    def fetch(self, idx_host: torch.Tensor, stream=None) -> MoeCacheStats:
        """Makes the experts of ``idx_host`` (int32 [T][top_k] on the host)
        resident; returns this call's hits, misses and copied bytes."""
        idx_host = idx_host.contiguous()
        if idx_host.is_cuda or idx_host.dtype != torch.int32:
            raise ValueError("idx_host: expected an int32 host tensor")
        st = MoeCacheStats()
        _check(lib.moe_cache_fetch(ctypes.byref(self.cfg), ctypes.byref(self.c), idx_host.data_ptr(),
                                   idx_host.shape[0], _stream(stream), ctypes.byref(st)), "moe_cache_fetch")
        return st


# ---------------------------------------------------------------------------
# entry points (same names as the C ABI)
# ---------------------------------------------------------------------------
def moe_workspace_bytes(cfg: MoeConfig, max_tokens: int) -> int:
    n = lib.moe_workspace_bytes(ctypes.byref(cfg), max_tokens)
    if n == 0:
        raise MoeError(MOE_EINVAL, "moe_workspace_bytes", lib.moe_last_error().decode())
    return n


def moe_workspace_init(ws: torch.Tensor, stream=None):
    _check(lib.moe_workspace_init(_ptr(ws, torch.uint8, name="ws"), ws.numel(), _stream(stream)),
           "moe_workspace_init")


def workspace(cfg: MoeConfig, max_tokens: int, device="cuda") -> torch.Tensor:
    """Allocate (through torch) and initialise a workspace for up to max_tokens."""
    ws = torch.empty(moe_workspace_bytes(cfg, max_tokens), dtype=torch.uint8, device=device)
    moe_workspace_init(ws)
    return ws


def moe_quantize(cfg: MoeConfig, x: torch.Tensor, xq: torch.Tensor, sx: torch.Tensor, stream=None):
    T = x.shape[0]
    _check(lib.moe_quantize(ctypes.byref(cfg), _ptr(x, name="x"), _xdtype(x), T,
                            _ptr(xq, torch.int8, T * cfg.d, "xq"), _ptr(sx, torch.float32, T, "sx"),
                            _stream(stream)), "moe_quantize")


def moe_route(cfg: MoeConfig, x: torch.Tensor, w_router: torch.Tensor, bias: torch.Tensor,
              topk_idx: torch.Tensor, topk_w: torch.Tensor, ws: torch.Tensor, stream=None):
    T = x.shape[0]
    _check(lib.moe_route(ctypes.byref(cfg), _ptr(x, name="x"), _xdtype(x), T,
                         _ptr(w_router, torch.float32, cfg.n_experts * cfg.d, "w_router"),
                         _ptr(bias, torch.float32, cfg.n_experts, "bias"),
                         _ptr(topk_idx, torch.int32, T * cfg.top_k, "topk_idx"),
                         _ptr(topk_w, torch.float32, T * cfg.top_k, "topk_w"),
                         _ptr(ws, torch.uint8, name="ws"), ws.numel(), _stream(stream)), "moe_route")


def moe_route_static(cfg: MoeConfig, x: torch.Tensor, w_router: torch.Tensor, bias: torch.Tensor,
                     topk_idx: torch.Tensor, topk_w: torch.Tensor, stream=None):
    """moe_route without a workspace, for callers that cannot allocate device
    memory on their call path; its scratch is a fixed array inside libmoe.so.
    Up to 8 tokens per call; calls that overlap on the GPU race."""
    T = x.shape[0]
    _check(lib.moe_route_static(ctypes.byref(cfg), _ptr(x, name="x"), _xdtype(x), T,
                                _ptr(w_router, torch.float32, cfg.n_experts * cfg.d, "w_router"),
                                _ptr(bias, torch.float32, cfg.n_experts, "bias"),
                                _ptr(topk_idx, torch.int32, T * cfg.top_k, "topk_idx"),
                                _ptr(topk_w, torch.float32, T * cfg.top_k, "topk_w"), _stream(stream)),
           "moe_route_static")


def moe_expert_ffn(cfg: MoeConfig, pool: MoePool, expert: int, xq: torch.Tensor, sx: torch.Tensor,
                   y: torch.Tensor, ws: torch.Tensor, dbg_acc_gu=None, dbg_hq=None, dbg_sh=None,
                   dbg_acc_d=None, stream=None):
    T = xq.shape[0]
    _check(lib.moe_expert_ffn(ctypes.byref(cfg), ctypes.byref(pool), expert,
                              _ptr(xq, torch.int8, T * cfg.d, "xq"), _ptr(sx, torch.float32, T, "sx"), T,
                              _ptr(y, torch.float32, T * cfg.d, "y"),
                              _ptr(dbg_acc_gu, torch.int32, T * 2 * cfg.f, "dbg_acc_gu"),
                              _ptr(dbg_hq, torch.int8, T * cfg.f, "dbg_hq"),
                              _ptr(dbg_sh, torch.float32, T, "dbg_sh"),
                              _ptr(dbg_acc_d, torch.int32, T * cfg.d, "dbg_acc_d"),
                              _ptr(ws, torch.uint8, name="ws"), ws.numel(), _stream(stream)), "moe_expert_ffn")


def moe_expert_down(cfg: MoeConfig, pool: MoePool, expert: int, hq: torch.Tensor, sh: torch.Tensor,
                    y: torch.Tensor, ws: torch.Tensor, dbg_acc_d=None, stream=None):
    T = hq.shape[0]
    _check(lib.moe_expert_down(ctypes.byref(cfg), ctypes.byref(pool), expert,
                               _ptr(hq, torch.int8, T * cfg.f, "hq"), _ptr(sh, torch.float32, T, "sh"), T,
                               _ptr(y, torch.float32, T * cfg.d, "y"),
                               _ptr(dbg_acc_d, torch.int32, T * cfg.d, "dbg_acc_d"),
                               _ptr(ws, torch.uint8, name="ws"), ws.numel(), _stream(stream)), "moe_expert_down")


def moe_layer(cfg: MoeConfig, pool: MoePool, w_router: torch.Tensor, bias: torch.Tensor, x: torch.Tensor,
              out: torch.Tensor, ws: torch.Tensor, accumulate: bool = False, topk_idx_out=None,
              topk_w_out=None, stream=None, opts: Optional[MoeLayerOpts] = None):
    """moe_layer, or moe_layer_ex when ``opts`` is given."""
    T = x.shape[0]
    io = opts.io_host if opts is not None else 0
    args = (ctypes.byref(cfg), ctypes.byref(pool),
            _ptr(w_router, torch.float32, cfg.n_experts * cfg.d, "w_router"),
            _ptr(bias, torch.float32, cfg.n_experts, "bias"), _ptr(x, name="x", host=bool(io & MOE_IO_X_HOST)),
            _xdtype(x), T,
            _ptr(out, torch.float32, T * cfg.d, "out", host=bool(io & MOE_IO_OUT_HOST)), 1 if accumulate else 0,
            _ptr(topk_idx_out, torch.int32, T * cfg.top_k, "topk_idx_out"),
            _ptr(topk_w_out, torch.float32, T * cfg.top_k, "topk_w_out"),
            _ptr(ws, torch.uint8, name="ws"), ws.numel(), _stream(stream))
    if opts is None:
        _check(lib.moe_layer(*args), "moe_layer")
    else:
        _check(lib.moe_layer_ex(*args, ctypes.byref(opts)), "moe_layer_ex")


def moe_rmsnorm(x: torch.Tensor, x_in: torch.Tensor, eps: float = 1e-6, x_copy=None, stream=None):
    T, d = x.shape
    _check(lib.moe_rmsnorm(_ptr(x, name="x"), _xdtype(x), T, d, eps, _ptr(x_in, torch.float32, T * d, "x_in"),
                           _ptr(x_copy, torch.float32, T * d, "x_copy"), _stream(stream)), "moe_rmsnorm")


def moe_poll_status(ws: torch.Tensor, stream=None) -> int:
    info = ctypes.c_int32(0)
    st = lib.moe_poll_status(_ptr(ws, torch.uint8, name="ws"), ctypes.byref(info), _stream(stream))
    return st


__all__ = [n for n in dir() if n.startswith("moe_")] + ["MoeConfig", "MoePool", "MoeLayerOpts", "MoeError", "config",
                                                         "make_pool", "workspace", "lib"]
