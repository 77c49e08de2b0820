"""The precision argument of the 3xTF32 routing kernels, checked on the CPU.

For fp32 means the routing kernels form each product x*y on the tensor cores as
hi(x)hi(y) + hi(x)lo(y) + lo(x)hi(y), where hi = tf32(x) rounds x to 10 explicit mantissa bits
(to nearest, ties away from zero) and lo = tf32(x - hi). The claims are:
  * x - hi is exact in fp32 and |x - hi - lo| <= 2^-22 |x|;
  * the three kept products (each exact in fp32: 11 x 11 significant bits) give a dot
    product within about 1e-6 of the sum of the terms' magnitudes, ten times inside the
    routing tolerance of 1e-5 (before the fp32 accumulation any summation order adds);
  * equal inputs give equal results (the split is a function of the value alone).
tf32 rounding is emulated here from its definition on fp32 bit patterns.
"""
import numpy as np

TOL_SPLIT = 2.0 ** -22
TOL_DOT = 1e-6


def tf32(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to tf32 (10 explicit mantissa bits), to nearest, ties away from zero."""
    u = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x1000) & 0xFFFFE000  # the sign bit is apart: this rounds the magnitude half up
    return u.astype(np.uint32).view(np.float32)


def split(x: np.ndarray):
    x = np.asarray(x, np.float32)
    hi = tf32(x)
    r = (x - hi).astype(np.float32)
    return hi, tf32(r), r


def _values(rng, n):
    # magnitudes over many binades, both signs, plus values near powers of two
    mag = np.exp2(rng.uniform(-20, 20, n)).astype(np.float32)
    x = (mag * rng.choice([-1.0, 1.0], n)).astype(np.float32)
    edges = np.exp2(np.arange(-10, 11)).astype(np.float32)
    return np.concatenate([x, edges, -edges, np.nextafter(edges, np.float32(0)), np.nextafter(edges, np.float32(np.inf))])


def test_tf32_rounding_matches_its_definition():
    # 1 + k 2^-10 are tf32 values; halfway points round away from zero
    step = 2.0 ** -10
    for k in range(0, 8):
        v = np.float32(1 + k * step)
        assert tf32(v) == v
        half = np.float32(1 + (k + 0.5) * step)
        assert tf32(half) == np.float32(1 + (k + 1) * step)
        assert tf32(-half) == -np.float32(1 + (k + 1) * step)
    # just below and above a halfway point
    h = np.float32(1 + 0.5 * step)
    assert tf32(np.nextafter(h, np.float32(0))) == np.float32(1)
    assert tf32(np.nextafter(h, np.float32(2))) == np.float32(1 + step)
    # the low 13 bits of every result are zero
    rng = np.random.Generator(np.random.PCG64(11))
    assert np.all(tf32(_values(rng, 4096)).view(np.uint32) & 0x1FFF == 0)


def test_split_is_exact_to_2_pow_minus_22():
    rng = np.random.Generator(np.random.PCG64(12))
    x = _values(rng, 1 << 16)
    hi, lo, r = split(x)
    x64, hi64, lo64 = x.astype(np.float64), hi.astype(np.float64), lo.astype(np.float64)
    assert np.all(r.astype(np.float64) == x64 - hi64), "x - hi must be exact in fp32"
    err = np.abs(x64 - hi64 - lo64)
    assert np.all(err <= TOL_SPLIT * np.abs(x64)), float(np.max(err / np.abs(x64)))
    # tf32 x tf32 products are exact in fp32 (11 x 11 significant bits fit in 24)
    p = (hi[:-1] * hi[1:]).astype(np.float64)
    assert np.all(p == hi64[:-1] * hi64[1:])


def test_three_products_give_dot_products_within_1e_6_of_their_terms():
    rng = np.random.Generator(np.random.PCG64(13))
    worst = 0.0
    for C in (64, 128, 256, 512):
        for _ in range(200):
            # means of N(0,1) tokens plus a region offset: the values routing sees
            x = (rng.normal(0, 1, C) / 8 + rng.normal(0, 0.5, C)).astype(np.float32)
            y = (rng.normal(0, 1, C) / 8 + rng.normal(0, 0.5, C)).astype(np.float32)
            hx, lx, _ = split(x)
            hy, ly, _ = split(y)
            h64x, l64x, h64y, l64y = (a.astype(np.float64) for a in (hx, lx, hy, ly))
            three = np.sum(l64x * h64y + h64x * l64y + h64x * h64y)
            exact = np.dot(x.astype(np.float64), y.astype(np.float64))
            mag = np.sum(np.abs(x.astype(np.float64) * y.astype(np.float64)))
            worst = max(worst, abs(three - exact) / mag)
    assert worst <= TOL_DOT, worst
    # dropping lo*lo is what keeps it above plain fp32: plain tf32 would be about 1e-3 off
    x = (rng.normal(0, 1, 256)).astype(np.float32)
    y = (rng.normal(0, 1, 256)).astype(np.float32)
    plain = np.dot(tf32(x).astype(np.float64), tf32(y).astype(np.float64))
    exact = np.dot(x.astype(np.float64), y.astype(np.float64))
    mag = np.sum(np.abs(x.astype(np.float64) * y.astype(np.float64)))
    assert abs(plain - exact) / mag > 10 * TOL_DOT


def test_equal_values_split_equally():
    rng = np.random.Generator(np.random.PCG64(14))
    x = _values(rng, 1024)
    a, b = split(x), split(x.copy())
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
