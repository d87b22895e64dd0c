"""fp32 identities the CUDA kernels rely on, checked with numpy's fp32.

- Head sums: w * max(x, 0) and (w / 2) * (x + |x|) are the same real number
  (x + |x| is exactly 2x or +0, w / 2 is exact for normal w), so they round
  to the same fp32 value, alone or inside an FMA.  The exceptions are the
  ones the kernels document: subnormal w (w / 2 rounds), |x| >= 2^127
  (x + |x| overflows) and NaN.
- DoSA screen: w max(d, 0) + a |d| = (w/2) d + (w/2 + a) |d| in exact
  arithmetic (the bound's slack absorbs the fp32 rounding of the rewrite).
- Final selection: the bucket digit min(2047, trunc((s - smin) * scale)) never
  decreases along the score order, which keeps the counting selection exact.
"""

import numpy as np

f32 = np.float32


def _random_f32(rng, n):
    mant = rng.standard_normal(n)
    expo = rng.integers(-60, 60, n).astype(np.float64)
    return (mant * 2.0 ** expo).astype(f32)


def test_halved_weight_times_x_plus_abs_x_equals_weighted_relu():
    rng = np.random.default_rng(0)
    x = np.concatenate([_random_f32(rng, 200000), np.array([0.0, -0.0, 1e-45, -1e-45, 3e38, -3e38], f32)])
    w = np.concatenate([_random_f32(rng, 200000), np.array([1.0, -1.0, 0.5, -2.0, 1e-30, 7.0], f32)])
    with np.errstate(over="ignore", invalid="ignore"):
        lhs = (w * f32(0.5)) * (x + np.abs(x))
        rhs = w * np.maximum(x, f32(0.0))
    normal_w = np.abs(w) >= f32(2.0 ** -125)  # w / 2 stays normal: exact halving
    finite_2x = np.abs(x) < f32(2.0 ** 127)
    ok = normal_w & finite_2x
    assert ok.sum() > 190000
    # bit for bit, signed zeros included (both are w times +0)
    assert np.array_equal(lhs[ok].view(np.uint32), rhs[ok].view(np.uint32))


def test_screen_bound_rewrite_is_exact_in_real_arithmetic():
    rng = np.random.default_rng(1)
    d = rng.standard_normal(100000) * 10.0
    w = rng.standard_normal(100000)
    a = np.abs(rng.standard_normal(100000))
    lhs = w * np.maximum(d, 0.0) + a * np.abs(d)
    rhs = (w / 2) * d + (w / 2 + a) * np.abs(d)
    scale = np.abs(w) * np.abs(d) + a * np.abs(d)
    assert np.all(np.abs(lhs - rhs) <= 1e-14 * scale + 1e-300)


def test_linear_score_digit_is_monotone():
    rng = np.random.default_rng(2)
    for trial in range(20):
        s = np.sort(_random_f32(rng, 5000) / f32(2.0 ** rng.integers(0, 40)))
        smin, smax = s[0], s[-1]
        srange = f32(smax - smin)
        if not (np.isfinite(srange) and srange > 0):
            continue
        scale = f32(2047.0) / srange
        if not np.isfinite(scale):
            continue
        with np.errstate(over="ignore"):
            prod = (s - smin).astype(f32) * scale
        digit = np.minimum(2047, np.trunc(prod).astype(np.float64)).astype(np.int64)
        assert digit.min() == 0 and digit.max() <= 2047
        assert np.all(np.diff(digit) >= 0)
