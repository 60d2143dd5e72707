"""Pins of the CPU oracle against things other than itself.

Each test checks the oracle against a hand-worked value, a closed form, an
invariant, a library routine the step reduces to, or brute force on tiny
inputs, so that a dropped term, a wrong sign or index, a transposed operand, a
swapped gate/up, a bias leaking into the weights or a wrong tie-break fails at
least one of them.
"""
import math

import numpy as np
import pytest

import oracle as O


# --------------------------------------------------------------------------
# helpers written independently of the oracle
# --------------------------------------------------------------------------
def pack_codes(wbits, codes):
    """Two's complement codes packed low bits first (int4: c0 | c1<<4)."""
    per = 8 // wbits
    codes = np.asarray(codes, np.int64).reshape(-1)
    assert codes.size % per == 0
    out = np.zeros(codes.size // per, np.uint8)
    for i, c in enumerate(codes):
        out[i // per] |= (int(c) & ((1 << wbits) - 1)) << ((i % per) * wbits)
    return out


def unpack_np(wbits, packed, n):
    per = 8 // wbits
    b = np.asarray(packed, np.uint8)
    out = np.empty(n, np.int64)
    for i in range(n):
        v = (int(b[i // per]) >> ((i % per) * wbits)) & ((1 << wbits) - 1)
        out[i] = v - (1 << wbits) if v >= (1 << (wbits - 1)) else v
    return out


# --------------------------------------------------------------------------
# packing
# --------------------------------------------------------------------------
@pytest.mark.parametrize("wbits", [4, 2, 8])
def test_pack_unpack_roundtrip_every_code_every_position(wbits):
    lo, hi = -(1 << (wbits - 1)), (1 << (wbits - 1)) - 1
    per = 8 // wbits
    codes = []
    for c in range(lo, hi + 1):
        for pos in range(per):
            grp = [0] * per
            grp[pos] = c
            codes += grp
    codes = np.array(codes, np.int8)
    packed = O.pack(wbits, codes)
    np.testing.assert_array_equal(packed, pack_codes(wbits, codes))
    np.testing.assert_array_equal(O.unpack(wbits, packed, codes.size), codes)


def test_unpack_hand_bytes():
    # int4: 0x8F -> low nibble 0xF = -1 first, high nibble 0x8 = -8 second
    np.testing.assert_array_equal(O.unpack(4, np.array([0x8F, 0x71], np.uint8), 4), [-1, -8, 1, 7])
    # int2: 0xE4 = 0b11_10_01_00 -> crumbs low first: 0, 1, -2, -1
    np.testing.assert_array_equal(O.unpack(2, np.array([0xE4], np.uint8), 4), [0, 1, -2, -1])
    # int8: one two's-complement code per byte
    np.testing.assert_array_equal(O.unpack(8, np.array([0x80, 0xFF, 0x00, 0x7F], np.uint8), 4), [-128, -1, 0, 127])


# --------------------------------------------------------------------------
# a0 quantiser
# --------------------------------------------------------------------------
def test_quantize_unit_scale_half_points_round_to_even():
    x = np.array([[127.0, 0.5, 1.5, 2.5, -0.5, -1.5, 126.5, -127.0]], np.float32)
    q, s = O.quantize(x)
    assert s[0] == 1.0
    np.testing.assert_array_equal(q[0], [127, 0, 2, 2, 0, -2, 126, -127])


def test_quantize_scale_and_extremes():
    x = np.array([[1.0, -1.0, 0.25, 0.0]], np.float32)
    q, s = O.quantize(x)
    assert s[0] == np.float32(1.0) / np.float32(127.0)
    # 0.25 * 127 = 31.75 -> 32
    np.testing.assert_array_equal(q[0], [127, -127, 32, 0])


def test_quantize_zero_token():
    q, s = O.quantize(np.zeros((2, 16), np.float32))
    assert (q == 0).all() and (s == 0).all()


def test_quantize_invariants_random():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((64, 96)).astype(np.float32) * rng.uniform(0.01, 100, (64, 1)).astype(np.float32)
    q, s = O.quantize(x)
    assert (np.abs(q.astype(int)) <= 127).all()
    assert (np.abs(q.astype(int)).max(axis=1) == 127).all()
    err = np.abs(q * s[:, None].astype(np.float64) - x)
    assert (err <= 0.5 * s[:, None] * (1 + 1e-5)).all()


# --------------------------------------------------------------------------
# a1 router
# --------------------------------------------------------------------------
L3 = math.log(3.0)


def hand_router():
    """d = 8, E = 4.  logit_e = 127*(W[e,0] - W[e,7]) on x = +-[127, 0.., -127]."""
    wr = np.zeros((4, 8), np.float32)
    wr[1, 0], wr[1, 7] = L3 / 254, -L3 / 254     # expert 1: logit +ln3 on token 0
    wr[2, 0], wr[2, 7] = -L3 / 254, L3 / 254     # expert 2: logit -ln3 on token 0
    bias = np.array([0.0, 0.0, 0.6, 0.0], np.float32)
    x = np.zeros((3, 8), np.float32)
    x[0, 0], x[0, 7] = 127.0, -127.0
    x[2, 0], x[2, 7] = -127.0, 127.0              # token 1 stays all-zero
    return x, wr, bias


def test_router_hand_case():
    x, wr, bias = hand_router()
    idx, w, lg, s, sel = O.route(x, wr, bias, k=2, routed_scale=2.5, want_scores=True)
    # token 0: s = [1/2, 3/4, 1/4, 1/2], sel = [.5, .75, .85, .5] -> experts 2 then 1;
    #          weights use the unbiased scores: 2.5*[.25, .75]/1.0
    # token 1: every s = 1/2, sel = [.5, .5, 1.1, .5] -> 2, then the tie {0,1,3} -> 0
    # token 2: s = [1/2, 1/4, 3/4, 1/2], sel = [.5, .25, 1.35, .5] -> 2, then tie {0,3} -> 0
    np.testing.assert_array_equal(idx, [[2, 1], [2, 0], [2, 0]])
    np.testing.assert_allclose(w, [[0.625, 1.875], [1.25, 1.25], [1.5, 1.0]], rtol=1e-6)
    np.testing.assert_allclose(s[0], [0.5, 0.75, 0.25, 0.5], rtol=1e-6)


def brute_topk(sel, k):
    order = sorted(range(len(sel)), key=lambda e: (-float(sel[e]), e))
    return order[:k]


@pytest.mark.parametrize("E,k,d,T", [(8, 2, 16, 7), (16, 5, 24, 9), (6, 6, 8, 3), (33, 8, 40, 5)])
def test_router_bruteforce_and_invariants(E, k, d, T):
    rng = np.random.default_rng(E * 100 + k)
    x = rng.standard_normal((T, d)).astype(np.float32)
    wr = (0.3 * rng.standard_normal((E, d))).astype(np.float32)
    # coarse bias values make exact ties in sel common
    bias = (rng.integers(-2, 3, E) * 0.125).astype(np.float32)
    idx, w, lg, s, sel = O.route(x, wr, bias, k, 2.5, want_scores=True)
    ref_logits = x.astype(np.float64) @ wr.astype(np.float64).T
    np.testing.assert_allclose(lg, ref_logits, rtol=1e-5, atol=1e-6)
    for t in range(T):
        assert list(idx[t]) == brute_topk(sel[t], k)
        np.testing.assert_allclose(w[t].sum(), 2.5, rtol=1e-12)
        st = s[t, idx[t]].astype(np.float64)
        np.testing.assert_allclose(w[t], 2.5 * st / st.sum(),
                                   rtol=1e-12)
    # sigmoid is monotone: with zero bias the selection is the top-k of the logits
    idx0, _ = O.route(x, wr, np.zeros(E, np.float32), k, 2.5)
    for t in range(T):
        assert set(idx0[t].tolist()) == set(np.argsort(-ref_logits[t], kind="stable")[:k].tolist())


def test_router_exact_ties_pick_lower_index():
    E, d = 8, 4
    wr = np.zeros((E, d), np.float32)  # every logit 0, every score 1/2
    bias = np.array([0, 0.1, 0, 0.1, 0, 0.1, 0, 0], np.float32)
    idx, w = O.route(np.ones((1, d), np.float32), wr, bias, 4, 1.0)
    np.testing.assert_array_equal(idx[0], [1, 3, 5, 0])
    np.testing.assert_allclose(w[0], [0.25] * 4)


# --------------------------------------------------------------------------
# a3/a4 integer dots: exact identities against int64 matmul of unpacked codes
# --------------------------------------------------------------------------
@pytest.mark.parametrize("wbits,d,f,T", [(4, 64, 32, 3), (2, 64, 48, 2), (4, 96, 40, 1), (8, 64, 32, 2)])
def test_expert_integer_identities(wbits, d, f, T):
    rng = np.random.default_rng(wbits * 1000 + d)
    blob = rng.integers(0, 256, 3 * d * f * wbits // 8, dtype=np.uint8)
    sc = np.exp(-4 + 0.3 * rng.standard_normal(2 * f + d)).astype(np.float32)
    x = rng.standard_normal((T, d)).astype(np.float32)
    xq, sx = O.quantize(x)
    r = O.expert(d, f, wbits, blob, sc, xq, sx)
    codes = unpack_np(wbits, blob, 3 * d * f)
    Wg = codes[: f * d].reshape(f, d)
    Wu = codes[f * d: 2 * f * d].reshape(f, d)
    Wd = codes[2 * f * d:].reshape(d, f)
    np.testing.assert_array_equal(r["acc_gu"][:, :f], xq.astype(np.int64) @ Wg.T)
    np.testing.assert_array_equal(r["acc_gu"][:, f:], xq.astype(np.int64) @ Wu.T)
    np.testing.assert_array_equal(r["acc_d"], r["hq"].astype(np.int64) @ Wd.T)
    # dequantised float dot / (s_row * s_x) reproduces the integer exactly
    deq = (Wg * sc[:f, None].astype(np.float64)) @ (xq[0].astype(np.float64) * float(sx[0]))
    np.testing.assert_allclose(deq / (sc[:f].astype(np.float64) * float(sx[0])), r["acc_gu"][0, :f],
                               rtol=1e-12, atol=1e-6)
    # y is the dequantised down accumulator
    np.testing.assert_allclose(r["y"], r["acc_d"] * sc[2 * f:][None, :].astype(np.float64) *
                               r["sh"][:, None].astype(np.float64), rtol=1e-15)
    # the teacher-forced down entry agrees with the fused one
    rd = O.down(d, f, wbits, blob, sc, r["hq"], r["sh"])
    np.testing.assert_array_equal(rd["acc_d"], r["acc_d"])


def test_expert_zero_token_and_zero_gate():
    d, f = 32, 8
    rng = np.random.default_rng(5)
    blob = rng.integers(0, 256, 3 * d * f // 2, dtype=np.uint8)
    sc = np.ones(2 * f + d, np.float32)
    r = O.expert(d, f, 4, blob, sc, np.zeros((1, d), np.int8), np.zeros(1, np.float32))
    assert (r["h"] == 0).all() and (r["y"] == 0).all() and r["sh"][0] == 0
    # gate codes all zero -> g = 0 -> SiLU(0) = 0 -> h = 0 whatever up is
    codes = unpack_np(4, blob, 3 * d * f)
    codes[: f * d] = 0
    blob0 = pack_codes(4, codes)
    xq, sx = O.quantize(rng.standard_normal((1, d)).astype(np.float32))
    r = O.expert(d, f, 4, blob0, sc, xq, sx)
    assert (r["h"] == 0).all() and (r["y"] == 0).all()


# --------------------------------------------------------------------------
# full layer, hand-worked: d = 8, f = 4, E = 4 routed + 1 shared, top-2, int4
# --------------------------------------------------------------------------
# Expert e: gate row r has code a at column 0 and code b at column 7; up row r
# has code c at column 0; every gate/up scale is 1/127.  With x = [127,0..,-127]
# (s_x = 1, xq = x) this gives G = 127(a-b), U = 127c, g = a-b, u = c; the
# opposite token gives g = b-a, u = -c.  Down rows 0..3: code 1 at column r;
# rows 4..7: code 2 at column r-4 and -1 at column (r-3) mod 4, so
# D[r] = hq[r] (r < 4) and D[r] = 2 hq[r-4] - hq[(r-3)%4] (r >= 4).
HAND_GATE = {0: [(1, 0), (0, 1), (2, 0), (0, 0)], 1: [(2, 0), (1, 1), (0, 2), (1, 0)],
             2: [(0, 1), (1, 0), (3, 1), (0, 0)], 3: [(1, 1), (0, 0), (1, 0), (0, 1)],
             4: [(1, 0), (1, 0), (1, 0), (1, 0)]}
HAND_UP = {0: [1, 2, -1, 3], 1: [1, 1, 1, -2], 2: [2, -1, 1, 1], 3: [1, 1, 1, 1], 4: [1, -1, 3, 0]}
HAND_SD = {0: [1.0] * 8, 1: [1, 1, 1, 1, .5, .5, .5, .5], 2: [.25] * 8, 3: [1.0] * 8, 4: [2.0] * 8}


def hand_pool():
    d, f = 8, 4
    blobs, scales = [], []
    for e in range(5):
        g = np.zeros((f, d), np.int64)
        u = np.zeros((f, d), np.int64)
        for r, (a, b) in enumerate(HAND_GATE[e]):
            g[r, 0], g[r, 7] = a, b
            u[r, 0] = HAND_UP[e][r]
        dn = np.zeros((d, f), np.int64)
        for r in range(d):
            if r < 4:
                dn[r, r] = 1
            else:
                dn[r, r - 4] += 2
                dn[r, (r - 3) % 4] += -1
        blobs.append(pack_codes(4, np.concatenate([g.ravel(), u.ravel(), dn.ravel()])))
        scales.append(np.array([1 / 127] * 8 + HAND_SD[e], np.float32))
    return blobs, scales


# silu(1) = 0.7310585786, silu(2) = 1.7615941560, silu(-1) = -0.2689414214,
# silu(-2) = -0.2384058440.
# token 0 selects experts (2, 1) with weights (0.625, 1.875), see the router case.
#  e2: g = [-1, 1, 2, 0], u = [2, -1, 1, 1]; h = [-0.53788, -0.73106, 1.76159, 0]
#      s_h = 1.76159/127; hq = rne(h/s_h) = [rne(-38.778), rne(-52.705), 127, 0]
#      = [-39, -53, 127, 0]; D = [-39, -53, 127, 0, -25, -233, 254, 39]; sd = 1/4
#  e1: g = [2, 0, -2, 1], u = [1, 1, 1, -2]; h = [1.76159, 0, -0.23841, -1.46212]
#      hq = [127, 0, rne(-17.188), rne(-105.410)] = [127, 0, -17, -105]
#      D = [127, 0, -17, -105, 254, 17, 71, -337]; sd = [1,1,1,1,.5,.5,.5,.5]
#  shared: g = [1,1,1,1], u = [1,-1,3,0]; h = [0.73106, -0.73106, 2.19318, 0]
#      hq = [rne(42.333), rne(-42.333), 127, 0] = [42, -42, 127, 0]
#      D = [42, -42, 127, 0, 126, -211, 254, -42]; sd = 2
# token 2 selects (2, 0) with weights (1.5, 1.0): every g and u flips sign.
#  e2: g = [1, -1, -2, 0], u = [-2, 1, -1, -1]; h = [-1.46212, -0.26894, 0.23841, 0]
#      hq = [-127, rne(-23.360), rne(20.708), 0] = [-127, -23, 21, 0]
#  e0: g = [-1, 1, -2, 0], u = [-1, -2, 1, -3]; h = [0.26894, -1.46212, -0.23841, 0]
#      hq = [23, -127, -21, 0]
#  shared: h = [0.26894, -0.26894, 0.80682, 0]; hq = [42, -42, 127, 0]
# out = sum_j w_j * D_j * sd_j * s_h_j + D_sh * sd_sh * s_h_sh.
HAND_OUT = {
    0: [4.669068156014742, -1.5654721529037001, 4.219468167143472, -2.730817712234576,
        7.600619422516125, -7.571478668703194, 10.246477581908877, -5.748391347040788],
    1: [0.0] * 8,
    2: [0.2501464817930002, -2.0950620286506108, 1.4625439007472334, 0.0,
        2.5953549922366115, -5.652667958048456, 2.925087801494467, -0.2501464817930002],
}
HAND_HQ = {(0, 2): [-39, -53, 127, 0], (0, 1): [127, 0, -17, -105], (0, 4): [42, -42, 127, 0],
           (2, 2): [-127, -23, 21, 0], (2, 0): [23, -127, -21, 0], (2, 4): [42, -42, 127, 0]}


def test_hand_layer():
    x, wr, bias = hand_router()
    blobs, scales = hand_pool()
    r = O.layer(8, 4, 4, 2, 1, 4, 2.5, blobs, scales, wr, bias, x)
    np.testing.assert_array_equal(r["idx"], [[2, 1], [2, 0], [2, 0]])
    np.testing.assert_array_equal(r["xq"][0], [127, 0, 0, 0, 0, 0, 0, -127])
    for t in range(3):
        np.testing.assert_allclose(r["out"][t], HAND_OUT[t], rtol=2e-6, atol=1e-9)
    for (t, e), hq in HAND_HQ.items():
        ex = O.expert(8, 4, 4, blobs[e], scales[e], r["xq"][t:t + 1], r["sx"][t:t + 1])
        np.testing.assert_array_equal(ex["hq"][0], hq)
        G = [127 * (a - b) * (1 if t == 0 else -1) for a, b in HAND_GATE[e]]
        np.testing.assert_array_equal(ex["acc_gu"][0, :4], G)


def test_layer_k_equals_E_is_plain_weighted_sum():
    """k = E, zero bias: every expert is selected; out = sum_e w_e y_e + y_shared
    with w_e = 2.5 s_e / sum s, whatever the selection order."""
    rng = np.random.default_rng(11)
    d, f, E = 32, 16, 4
    blobs = [rng.integers(0, 256, 3 * d * f // 2, dtype=np.uint8) for _ in range(E + 1)]
    scales = [np.exp(-4 + 0.3 * rng.standard_normal(2 * f + d)).astype(np.float32) for _ in range(E + 1)]
    wr = (0.2 * rng.standard_normal((E, d))).astype(np.float32)
    x = rng.standard_normal((2, d)).astype(np.float32)
    r = O.layer(d, f, E, E, 1, 4, 2.5, blobs, scales, wr, np.zeros(E, np.float32), x)
    _, _, _, s, _ = O.route(x, wr, np.zeros(E, np.float32), E, 2.5, want_scores=True)
    for t in range(2):
        acc = np.zeros(d)
        for e in range(E + 1):
            y = O.expert(d, f, 4, blobs[e], scales[e], r["xq"][t:t + 1], r["sx"][t:t + 1])["y"][0]
            we = 1.0 if e == E else 2.5 * float(s[t, e]) / s[t].astype(np.float64).sum()
            acc += we * y
        np.testing.assert_allclose(r["out"][t], acc, rtol=1e-12, atol=1e-12)


def test_layer_zero_token_is_zero():
    rng = np.random.default_rng(3)
    d, f, E = 32, 16, 4
    blobs = [rng.integers(0, 256, 3 * d * f // 2, dtype=np.uint8) for _ in range(E + 1)]
    scales = [np.ones(2 * f + d, np.float32)] * (E + 1)
    r = O.layer(d, f, E, 2, 1, 4, 2.5, blobs, scales, rng.standard_normal((E, d)).astype(np.float32),
                np.zeros(E, np.float32), np.zeros((1, d), np.float32))
    assert (r["out"] == 0).all()


def test_rmsnorm_closed_forms():
    x = np.array([[3.0] * 8, [-2.0, 2.0] * 4, [0.0] * 8])
    y = O.rmsnorm(x, eps=0.0 + 1e-6)
    np.testing.assert_allclose(y[0], [3 / math.sqrt(9 + 1e-6)] * 8, rtol=1e-7)
    np.testing.assert_allclose(y[1], [-2 / math.sqrt(4 + 1e-6), 2 / math.sqrt(4 + 1e-6)] * 4, rtol=1e-7)
    assert (y[2] == 0).all()


# --------------------------------------------------------------------------
# a1' TOPK/TOPP truncation (opt-in): smallest prefix of the selected slots
# whose normalised scores reach p, the rest dropped (idx -1, weight 0), the
# kept weights renormalised
# --------------------------------------------------------------------------
def test_topp_hand_cases():
    x, wr, _ = hand_router()
    bias = np.zeros(4, np.float32)
    # token 0: s = [1/2, 3/4, 1/4, 1/2] -> slots: experts 1, 0, 3, 2 with scores
    # .75, .5, .5, .25 (sum 2): prefixes before each slot 0, .75, 1.25, 1.75
    cases = {
        0.3: ([1, -1, -1, -1], [2.5, 0, 0, 0]),                       # thr .6: .75 >= .6 stops at 1 slot
        0.5: ([1, 0, -1, -1], [1.5, 1.0, 0, 0]),                      # thr 1.0: 1.25 stops at 2
        0.7: ([1, 0, 3, -1], [2.5 * .75 / 1.75, 2.5 * .5 / 1.75, 2.5 * .5 / 1.75, 0]),  # thr 1.4
        0.9: ([1, 0, 3, 2], [2.5 * .75 / 2, 2.5 * .5 / 2, 2.5 * .5 / 2, 2.5 * .25 / 2]),  # thr 1.8: all
        0.0: ([1, 0, 3, 2], [0.9375, 0.625, 0.625, 0.3125]),          # off
        1.0: ([1, 0, 3, 2], [0.9375, 0.625, 0.625, 0.3125]),          # off
    }
    for p, (want_idx, want_w) in cases.items():
        idx, w = O.route(x[:1], wr, bias, k=4, routed_scale=2.5, topp=p)
        np.testing.assert_array_equal(idx[0], want_idx, err_msg=str(p))
        np.testing.assert_allclose(w[0], want_w, rtol=1e-6, atol=0, err_msg=str(p))
    # token 1 (all scores exactly 1/2): at p = .5 the first two slots sum to
    # exactly p: the prefix that reaches p is kept, the next slot dropped
    idx, w = O.route(x[1:2], wr, bias, k=4, routed_scale=2.5, topp=0.5)
    np.testing.assert_array_equal(idx[0], [0, 1, -1, -1])
    np.testing.assert_allclose(w[0], [1.25, 1.25, 0, 0])


@pytest.mark.parametrize("E,k,d,T", [(16, 5, 24, 9), (33, 8, 40, 6)])
def test_topp_invariants(E, k, d, T):
    rng = np.random.default_rng(7 * E + k)
    x = rng.standard_normal((T, d)).astype(np.float32)
    wr = (0.5 * rng.standard_normal((E, d))).astype(np.float32)
    bias = (0.05 * rng.standard_normal(E)).astype(np.float32)
    full, wfull, _, s, _ = O.route(x, wr, bias, k, 2.5, want_scores=True)
    prev = np.ones(T, int)
    for p in (1e-6, 0.2, 0.4, 0.6, 0.8, 0.95):
        idx, w = O.route(x, wr, bias, k, 2.5, topp=p)
        for t in range(T):
            m = int((idx[t] >= 0).sum())
            assert m >= 1 and (idx[t][:m] >= 0).all() and (idx[t][m:] == -1).all()  # a kept prefix
            np.testing.assert_array_equal(idx[t][:m], full[t][:m])  # the selection order is untouched
            assert m >= prev[t]  # more slots as p grows
            prev[t] = m
            st = s[t, full[t]].astype(np.float64)
            q = np.cumsum(st) / st.sum()
            assert q[m - 1] >= p - 1e-6 and (m == 1 or q[m - 2] < p + 1e-6)  # the smallest prefix reaching p
            np.testing.assert_allclose(w[t][:m].sum(), 2.5, rtol=1e-12)
            np.testing.assert_allclose(w[t][:m], 2.5 * st[:m] / st[:m].sum(), rtol=1e-12)
            assert (w[t][m:] == 0).all()
        if p == 1e-6:
            assert (prev == 1).all()


def test_topp_layer_drops_the_truncated_experts():
    """The layer with truncation equals the weighted sum over the kept slots
    of the single-expert outputs (plus the shared expert)."""
    rng = np.random.default_rng(11)
    d, f, E, k, T, wb = 32, 16, 6, 4, 3, 4
    blobs = [rng.integers(0, 256, 3 * d * f * wb // 8, dtype=np.uint8) for _ in range(E + 1)]
    scales = [np.exp(-4 + 0.3 * rng.standard_normal(2 * f + d)).astype(np.float32) for _ in range(E + 1)]
    x = rng.standard_normal((T, d)).astype(np.float32)
    wr = (0.5 * rng.standard_normal((E, d))).astype(np.float32)
    bias = np.zeros(E, np.float32)
    r = O.layer(d, f, E, k, 1, wb, 2.5, blobs, scales, wr, bias, x, topp=0.55)
    idx, w = O.route(x, wr, bias, k, 2.5, topp=0.55)
    np.testing.assert_array_equal(r["idx"], idx)
    assert (idx == -1).any() and (idx >= 0).any()
    xq, sx = O.quantize(x)
    for t in range(T):
        want = O.expert(d, f, wb, blobs[E], scales[E], xq[t:t + 1], sx[t:t + 1])["y"][0].copy()
        for j in range(k):
            if idx[t, j] >= 0:
                want += w[t, j] * O.expert(d, f, wb, blobs[idx[t, j]], scales[idx[t, j]], xq[t:t + 1],
                                           sx[t:t + 1])["y"][0]
        np.testing.assert_allclose(r["out"][t], want, rtol=1e-12, atol=1e-12)
