"""The C ABI library without a GPU: it loads, exports every entry point the
header declares, sizes workspaces, and rejects bad arguments on the host
before launching anything (no call here reaches a kernel launch)."""
import ctypes

import pytest

import expert_ffn_router_b200 as M

L = M.lib
FAKE = 1 << 20  # 16-byte aligned fake device address (never dereferenced)


def good_cfg(**kw):
    c = M.config(128, 64, 8, 2, 1, 4, 2.5)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def test_exports_every_declared_symbol():
    names = M.declared_symbols()
    assert len(names) >= 11
    for n in names:
        assert hasattr(L, n), n
    for n in ("moe_route", "moe_expert_ffn", "moe_layer"):
        assert n in names


def test_workspace_bytes():
    c = good_cfg()
    n1 = M.moe_workspace_bytes(c, 1)
    n32 = M.moe_workspace_bytes(c, 32)
    assert 256 < n1 < n32
    big = M.config(6144, 2048, 256, 8, 1, 4)
    assert M.moe_workspace_bytes(big, 512) > 512 * 9 * 6144 * 4  # slot buffer of the combine
    assert L.moe_workspace_bytes(ctypes.byref(good_cfg(wbits=3)), 4) == 0


@pytest.mark.parametrize("field,value", [("wbits", 3), ("d", 100), ("f", 40), ("top_k", 0), ("top_k", 9),
                                         ("n_experts", 0), ("has_shared", 2), ("d", 16384), ("topp", -0.1),
                                         ("topp", 1.5), ("topp", float("nan"))])
def test_layer_rejects_bad_config(field, value):
    c = good_cfg(**{field: value})
    pool = M.MoePool(FAKE, FAKE)
    st = L.moe_layer(ctypes.byref(c), ctypes.byref(pool), FAKE, FAKE, FAKE, 0, 4, FAKE, 0, None, None, FAKE,
                     1 << 40, None)
    assert st == M.MOE_EINVAL
    assert L.moe_last_error()


def test_layer_rejects_misaligned_and_null_and_small_ws():
    c = good_cfg()
    pool = M.MoePool(FAKE, FAKE)
    args = lambda x=FAKE, ws=FAKE, wsb=1 << 40, out=FAKE: (ctypes.byref(c), ctypes.byref(pool), FAKE, FAKE, x, 0,
                                                             4, out, 0, None, None, ws, wsb, None)
    assert L.moe_layer(*args(x=FAKE + 4)) == M.MOE_EALIGN
    assert L.moe_layer(*args(out=None)) == M.MOE_EINVAL
    assert L.moe_layer(*args(wsb=1000)) == M.MOE_ENOSPACE
    assert L.moe_layer(ctypes.byref(c), None, FAKE, FAKE, FAKE, 0, 4, FAKE, 0, None, None, FAKE, 1 << 40,
                       None) == M.MOE_EINVAL
    assert L.moe_layer(*args()[:5], 7, *args()[6:]) == M.MOE_EINVAL  # bad dtype
    # T = 0 is a no-op and succeeds without touching the device
    a = list(args())
    a[6] = 0
    assert L.moe_layer(*a) == M.MOE_OK


def test_expert_entry_points_validate():
    c = good_cfg()
    pool = M.MoePool(FAKE, FAKE)
    st = L.moe_expert_ffn(ctypes.byref(c), ctypes.byref(pool), 8, FAKE, FAKE, 4, FAKE, None, None, None, None,
                          FAKE, 1 << 40, None)
    assert st == M.MOE_EINVAL  # expert out of range
    st = L.moe_expert_ffn(ctypes.byref(c), ctypes.byref(pool), -1, FAKE, FAKE, 4, FAKE, FAKE + 8, None, None,
                          None, FAKE, 1 << 40, None)
    assert st == M.MOE_EALIGN  # misaligned debug output
    c0 = good_cfg(has_shared=0)
    st = L.moe_expert_down(ctypes.byref(c0), ctypes.byref(pool), -1, FAKE, FAKE, 4, FAKE, None, FAKE, 1 << 40,
                           None)
    assert st == M.MOE_EINVAL  # no shared expert
    st = L.moe_route(ctypes.byref(c), FAKE, 0, -1, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 40, None)
    assert st == M.MOE_EINVAL
    assert L.moe_rmsnorm(FAKE, 0, 4, 30, 1e-6, FAKE, None, None) == M.MOE_EINVAL  # d not a multiple of 4


def test_status_strings():
    for st in (0, -1, -2, -3, -4, -5, -6):
        assert L.moe_status_string(st).decode().startswith("MOE_")


def test_bounds_checked_build_exports_the_same_symbols():
    import os
    path = os.path.join(os.path.dirname(M.LIB_PATH), "libmoe_bounds.so")
    assert os.path.exists(path), "libmoe_bounds.so is not built"
    B = ctypes.CDLL(path)
    for n in M.declared_symbols():
        assert hasattr(B, n), n


def test_layer_opts_rejects_negative_test_fields():
    c = good_cfg()
    pool = M.MoePool(FAKE, FAKE)
    o = M.MoeLayerOpts()
    o.wait_limit_us = -1
    st = L.moe_layer_ex(ctypes.byref(c), ctypes.byref(pool), FAKE, FAKE, FAKE, 0, 4, FAKE, 0, None, None, FAKE,
                        1 << 40, None, ctypes.byref(o))
    assert st == M.MOE_EINVAL
    o.wait_limit_us, o.test_skip_h = 0, -3
    st = L.moe_layer_ex(ctypes.byref(c), ctypes.byref(pool), FAKE, FAKE, FAKE, 0, 4, FAKE, 0, None, None, FAKE,
                        1 << 40, None, ctypes.byref(o))
    assert st == M.MOE_EINVAL
    o.test_skip_h, o.io_host = 0, 4  # an unknown io_host bit
    st = L.moe_layer_ex(ctypes.byref(c), ctypes.byref(pool), FAKE, FAKE, FAKE, 0, 4, FAKE, 0, None, None, FAKE,
                        1 << 40, None, ctypes.byref(o))
    assert st == M.MOE_EINVAL


def test_cache_entry_points_validate_on_the_host():
    c = good_cfg()
    assert L.moe_cache_state_bytes(ctypes.byref(c), 0) == 0
    n4 = L.moe_cache_state_bytes(ctypes.byref(c), 4)
    assert n4 > L.moe_cache_state_bytes(ctypes.byref(c), 2) > 0
    cache = M.MoeCache(FAKE, FAKE, FAKE, FAKE, 1)  # one slot cannot hold the shared expert and another
    assert L.moe_cache_init(ctypes.byref(c), ctypes.byref(cache), None) == M.MOE_EINVAL
    cache = M.MoeCache(None, FAKE, FAKE, FAKE, 4)
    assert L.moe_cache_init(ctypes.byref(c), ctypes.byref(cache), None) == M.MOE_EINVAL
    cache = M.MoeCache(FAKE, FAKE + 4, FAKE, FAKE, 4)  # slots not 16-byte aligned
    assert L.moe_cache_init(ctypes.byref(c), ctypes.byref(cache), None) == M.MOE_EALIGN
    # a fetch before init is refused (the state's header does not match)
    state = (ctypes.c_uint64 * (n4 // 8 + 1))()
    cache = M.MoeCache(FAKE, FAKE, FAKE, ctypes.addressof(state), 4)
    idx = (ctypes.c_int32 * 2)(0, 1)
    assert L.moe_cache_fetch(ctypes.byref(c), ctypes.byref(cache), ctypes.addressof(idx), 1, None, None) == \
        M.MOE_EINVAL
    # a pool with a slot table must say how many blobs it holds
    pool = M.MoePool(FAKE, FAKE, FAKE, 0)
    st = L.moe_layer(ctypes.byref(c), ctypes.byref(pool), FAKE, FAKE, FAKE, 0, 4, FAKE, 0, None, None, FAKE,
                     1 << 40, None)
    assert st == M.MOE_EINVAL
