"""The division-free quantiser the kernels use gives the same codes as the
layer's rule (IEEE quotient, round half to even, clamp to +-127).

The kernels compute q = fl(v * fl(1 / s)) and take the exact quotient only
when q lies within 1e-3 of a half-integer (or |q| > 128, or 1/s overflows).
Emulated here in float32 arithmetic, which numpy rounds exactly like the GPU's
fp32 multiply and divide, on random rows and on adversarial values placed at
and next to every half-point of the code range.
"""
import numpy as np

F32 = np.float32


def exact_codes(v, s):
    return np.clip(np.rint(v / s), -127, 127).astype(np.int32)


def fast_codes(v, s):
    with np.errstate(over="ignore", divide="ignore", invalid="ignore"):
        r = F32(1) / s
        q = (v * r).astype(F32)
        aq = np.abs(q)
        frac = aq - np.floor(aq)
        slow = ~(aq <= F32(128)) | (np.abs(frac - F32(0.5)) < F32(1e-3))
    out = np.clip(np.rint(q), -127, 127)
    out = np.where(slow, exact_codes(v, s), out)
    return out.astype(np.int32), int(slow.sum())


def scale_of(v):
    m = np.max(np.abs(v)).astype(F32)
    return (m / F32(127)).astype(F32)


def test_random_rows_match_the_exact_rule():
    rng = np.random.default_rng(1234)
    n_slow = n_all = 0
    for scale in (1e-3, 1.0, 37.0, 1e4):
        for _ in range(200):
            v = (rng.standard_normal(4096) * scale).astype(F32)
            v[rng.integers(0, 4096, 8)] *= F32(20)  # outlier channels
            s = scale_of(v)
            fc, ns = fast_codes(v, s)
            np.testing.assert_array_equal(fc, exact_codes(v, s))
            n_slow += ns
            n_all += v.size
    assert n_slow < 0.01 * n_all  # the exact fallback stays rare


def test_half_points_and_their_neighbours():
    """v placed at (k + 1/2) s and one float step either side, for every k."""
    rng = np.random.default_rng(7)
    for _ in range(50):
        m = F32(rng.uniform(1e-3, 1e3))
        s = (m / F32(127)).astype(F32)
        k = np.arange(-128, 128, dtype=np.float64)
        mid = ((k + 0.5) * np.float64(s)).astype(F32)
        v = np.concatenate([mid, np.nextafter(mid, np.float32(np.inf)), np.nextafter(mid, np.float32(-np.inf)),
                            np.array([m, -m, 0, -0.0], dtype=F32)]).astype(F32)
        v = np.clip(v, -m, m)  # a row's values never exceed its max
        fc, _ = fast_codes(v, s)
        np.testing.assert_array_equal(fc, exact_codes(v, s))


def test_extreme_scales():
    rng = np.random.default_rng(99)
    for m in (F32(1e-38), F32(3e-39), F32(1e-30), F32(3e38)):
        v = (rng.uniform(-1, 1, 2048) * m).astype(F32)
        v[0] = m
        s = (m / F32(127)).astype(F32)
        fc, _ = fast_codes(v, s)
        np.testing.assert_array_equal(fc, exact_codes(v, s))
