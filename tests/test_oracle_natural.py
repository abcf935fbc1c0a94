"""Pins of the oracle's natural compression (Horvath et al., "Natural Compression
for Distributed Deep Learning", cited in the Global-QSGD record).

Each test checks the oracle against something other than its own code: exact
powers of two, the two neighbouring powers computed here with math.frexp, the
integer carry test on raw Philox bits, Monte Carlo frequencies against the
closed-form probability and variance (and the published bound x^2/8), and fp32
sums that are exact or whose rounding is worked out by hand.
"""
import math

import numpy as np
import pytest


def brackets(x):
    """(lower, upper) powers of two around |x| (0 and 2^-126 below the normals)."""
    ax = abs(float(x))
    if ax < 2.0 ** -126:
        return 0.0, 2.0 ** -126
    m, e = math.frexp(ax)  # ax = m 2^e, m in [0.5, 1)
    return math.ldexp(1.0, e - 1), math.ldexp(1.0, e)


def test_powers_of_two_and_zeros_are_fixed(oracle):
    ks = np.arange(-126, 128)
    vals = np.concatenate([np.ldexp(1.0, ks), -np.ldexp(1.0, ks), [0.0, -0.0]]).astype(np.float32)
    x = np.tile(vals, (3, 1))
    for step in range(4):
        c = oracle.nat_quantize(x, seed=11, step=step)
        got = oracle.nat_decode(c)
        assert np.array_equal(got.view(np.uint32), x.view(np.uint32))
    assert oracle.nat_quantize(np.array([[0.0, -0.0]], np.float32))[0].tolist() == [0, 256]


def test_codes_are_sign_and_exponent():
    import oracle
    for code in (0, 1, 127, 128, 254, 256, 256 + 127, 256 + 1):
        E, neg = code & 0xFF, code >> 8
        want = 0.0 if E == 0 else math.ldexp(1.0, E - 127)
        v = oracle.nat_decode(np.array([code], np.uint16))[0]
        assert float(v) == (-want if neg else want)
        assert bool(np.signbit(v)) == bool(neg)


def test_every_result_is_one_of_the_two_neighbours(oracle):
    rng = np.random.default_rng(3)
    mags = np.ldexp(rng.uniform(1.0, 2.0, 4000), rng.integers(-140, 120, 4000))
    x = (mags * rng.choice([-1.0, 1.0], 4000)).astype(np.float32).reshape(4, 1000)
    got = oracle.nat_decode(oracle.nat_quantize(x, seed=5, step=1))
    for xv, gv in zip(x.ravel(), got.ravel()):
        lo, hi = brackets(xv)
        assert abs(float(gv)) in (lo, hi), (xv, gv)
        assert np.signbit(gv) == np.signbit(xv)


def test_decision_is_the_integer_carry(oracle):
    """Up exactly when mantissa field + top 23 Philox bits >= 2^23."""
    rng = np.random.default_rng(4)
    W, n = 3, 700
    x = (rng.standard_normal((W, n)) * np.ldexp(1.0, rng.integers(-20, 20, (W, n)))
         ).astype(np.float32)
    x[0, :5] = np.array([1e-40, -3e-39, 2.0 ** -126, 0.0, -0.0], np.float32)
    seed, step, worker0 = 0x123456789, 7, 5
    codes = oracle.nat_quantize(x, seed=seed, step=step, worker0=worker0)
    bits = x.view(np.uint32)
    for w in range(W):
        for i in range(n):
            f = oracle.uniform_bits(seed, oracle.NAT_TAG, step, worker0 + w, i)
            b = int(bits[w, i])
            assert int(codes[w, i]) == (b + f) >> 23, (w, i)


@pytest.mark.parametrize("x", [1.25, -3.0, 5.0 * 2.0 ** -60, 1.0 + 2.0 ** -10, 4.0 / 3.0])
def test_unbiased_with_closed_form_variance(oracle, x):
    """E[C(x)] = x and Var = (hi - |x|)(|x| - lo) <= x^2 / 8 (tight at p = 1/3)."""
    N = 40000
    xs = np.full((1, N), x, np.float32)
    lo, hi = brackets(np.float32(x))
    ax = abs(float(np.float32(x)))
    p = (ax - lo) / (hi - lo)
    # N coordinates of one step draw N different uniforms
    vals = np.abs(oracle.nat_decode(oracle.nat_quantize(xs, seed=9, step=3))[0].astype(np.float64))
    ups = vals == hi
    assert np.all((vals == hi) | (vals == lo))
    sd = math.sqrt(p * (1 - p) / N)
    assert abs(ups.mean() - p) <= 4 * sd + 1.0 / N
    var_closed = (hi - ax) * (ax - lo)
    assert var_closed <= ax * ax / 8 * (1 + 1e-12)
    # (C - x)^2 takes (hi - x)^2 with probability p and (x - lo)^2 otherwise:
    # its sample mean has standard error sqrt(p (1 - p) / N) |a - b|
    var_mc = float(np.mean((vals - ax) ** 2))
    a, b = (hi - ax) ** 2, (ax - lo) ** 2
    assert abs(var_mc - var_closed) <= 4 * math.sqrt(p * (1 - p) / N) * abs(a - b) + 1e-300
    if abs(p - 1.0 / 3.0) < 1e-6:
        assert abs(var_closed - ax * ax / 8) <= 1e-9 * ax * ax


def test_subnormals_round_between_zero_and_the_smallest_normal(oracle):
    x = np.full((1, 30000), 2.0 ** -130, np.float32)  # p = 2^-4
    vals = oracle.nat_decode(oracle.nat_quantize(x, seed=2, step=0))[0]
    assert set(np.unique(vals).tolist()) <= {0.0, 2.0 ** -126}
    freq = float(np.mean(vals > 0))
    assert abs(freq - 1 / 16) <= 4 * math.sqrt((1 / 16) * (15 / 16) / 30000)


def test_decode_sum_exact_when_fp32_is_exact(oracle):
    rng = np.random.default_rng(7)
    W, n = 8, 500
    E = rng.integers(127 - 8, 127 + 9, (W, n))
    sign = rng.integers(0, 2, (W, n))
    codes = (sign << 8 | E).astype(np.uint16)
    vals = np.ldexp(1.0, E - 127) * np.where(sign == 1, -1.0, 1.0)
    got = oracle.nat_decode_sum(codes)
    assert np.array_equal(got.astype(np.float64), vals.sum(axis=0))


def test_decode_sum_follows_the_worker_order(oracle):
    # 2^24 + 1 rounds back to 2^24 (ties to even), twice, then - 2^24 leaves 0;
    # the exact sum is 2.
    codes = np.array([[127 + 24], [127], [127], [256 + 127 + 24]], np.uint16)
    assert oracle.nat_decode_sum(codes)[0] == 0.0
    codes2 = np.array([[127], [127], [127 + 24], [256 + 127 + 24]], np.uint16)
    assert oracle.nat_decode_sum(codes2)[0] == 2.0


def test_worker_offset_selects_the_rows_stream(oracle):
    x = np.random.default_rng(1).standard_normal((5, 300)).astype(np.float32)
    full = oracle.nat_quantize(x, seed=3, step=4)
    part = oracle.nat_quantize(x[2:4], seed=3, step=4, worker0=2)
    assert np.array_equal(full[2:4], part)


def test_coordinate_list_selects_the_columns_stream(oracle):
    x = np.random.default_rng(2).standard_normal((3, 400)).astype(np.float32)
    full = oracle.nat_quantize(x, seed=6, step=1)
    js = np.array([0, 5, 7, 128, 399], np.int64)
    part = oracle.nat_quantize(x[:, js], seed=6, step=1, js=js)
    assert np.array_equal(full[:, js], part)

