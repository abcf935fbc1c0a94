"""Pins for the oracle's scale, quantizers, aggregation, decode and error feedback.

What the pages fix, and how each is checked here without re-typing the
oracle's own formulas:

* Unbiasedness ("Quantize Once, Train Fast", Abstract: the method extends the
  unbiased-compressor framework; "Unbiased Single-scale and Multi-scale
  Quantizers", title and Abstract): E[Q(x)] = x by Monte Carlo within 4 sigma,
  sigma from the Bernoulli closed form.
* QSGD variance (QSGD is the baseline named in the NUQSGD Abstract): the exact
  variance sum_j (S/s)^2 p_j (1 - p_j) is matched by Monte Carlo and is below
  min(d/s^2, sqrt(d)/s) * ||x||^2 when S = ||x||.
* Range and sign: |code| <= s (uniform) or <= L (exponential), sign kept.
* Inputs on a level are reproduced for every seed.
* Exact enumeration of the 2^3 rounding outcomes at d = 3, in rationals.
* Allreduce compatibility ("Quantize Once, Train Fast", Abstract; "Unbiased
  Single-scale and Multi-scale Quantizers", Abstract): the sum of the decoded
  codes equals the decoded sum of codes, exactly in fp64, with the level
  values taken from the level-set definition, not from the oracle.
* Error feedback (LQ-SGD review, "What carries the argument": E_t = G'_t -
  Ghat_t is added back next step): telescoping sum over steps.
"""
from fractions import Fraction
import itertools
import math

import numpy as np
import pytest

import synthetic

UNIFORM, EXP = 0, 1


# ----------------------------------------------------------------------------- scale
def test_l2_scale_matches_numpy_norm(oracle):
    g = synthetic.numpy_normal(5, 3001, 1) * np.float32(3.5)
    e = synthetic.numpy_normal(5, 3001, 2) * np.float32(0.1)
    S, norms = oracle.global_scale(g, e, oracle.SCALE_L2)
    v = (g + e).astype(np.float64)          # numpy's fp32 add, then widen
    ref = np.linalg.norm(v, axis=1)
    assert np.allclose(norms, ref, rtol=1e-13, atol=0)
    assert S == np.float32(ref.max())


def test_l2_scale_single_nonzero_is_exact(oracle):
    g = np.zeros((3, 100), np.float32)
    g[1, 37] = -1.2345678e-3
    S, _ = oracle.global_scale(g)
    assert S == np.float32(1.2345678e-3)


def test_maxabs_scale_is_exact_max(oracle):
    g = synthetic.numpy_normal(4, 999, 3)
    S, norms = oracle.global_scale(g, None, oracle.SCALE_MAXABS)
    assert S == np.abs(g).max()
    assert np.array_equal(norms, np.abs(g).max(axis=1).astype(np.float64))


def test_nan_input_gives_nan_scale(oracle):
    g = synthetic.numpy_normal(2, 50, 4)
    g[1, 3] = np.nan
    for kind in (oracle.SCALE_L2, oracle.SCALE_MAXABS):
        S, _ = oracle.global_scale(g, None, kind)
        assert np.isnan(S)


# ------------------------------------------------------------------ helpers (tests)
def level_value(code, levels, s, L, S):
    """Value of one code from the level-set definitions, as an exact Fraction."""
    k = abs(int(code))
    if levels == UNIFORM:
        mag = Fraction(k, s)
    else:
        mag = Fraction(0) if k == 0 else Fraction(2) ** (k - L)
    return (-mag if code < 0 else mag) * Fraction(float(S))


def bracket(x, levels, s, L, S):
    """(lower level, upper level, p) of |x|/S from the level definition, exact."""
    r = Fraction(abs(float(x))) / Fraction(float(S))
    if levels == UNIFORM:
        y = r * s
        lo = math.floor(y)
        return Fraction(lo, s), Fraction(min(lo + 1, s), s), y - lo
    finest = Fraction(1, 2 ** (L - 1))
    if r < finest:
        return Fraction(0), finest, r / finest
    e = math.floor(math.log2(r))
    while Fraction(2) ** e > r:
        e -= 1
    while Fraction(2) ** (e + 1) <= r:
        e += 1
    lo = Fraction(2) ** e
    if lo >= 1:
        return Fraction(1), Fraction(1), Fraction(0)
    return lo, 2 * lo, (r - lo) / lo


def replicas(x, N):
    return np.ascontiguousarray(np.broadcast_to(np.asarray(x, np.float32), (N, len(x))))


# ------------------------------------------------------------- T1 unbiasedness
@pytest.mark.parametrize("levels,s,L", [(UNIFORM, 15, 8), (UNIFORM, 3, 8), (EXP, 15, 8),
                                        (EXP, 15, 3)])
def test_unbiased_monte_carlo(oracle, levels, s, L):
    d, N = 16, 1 << 20
    x = synthetic.numpy_normal(1, d, 10)[0]
    x[3] = 0.0
    S = np.float32(np.linalg.norm(x.astype(np.float64)))
    # N replicas of the same vector: workers 0..N-1 draw independent uniforms
    codes = oracle.quantize(replicas(x, N), levels=levels, s=s, L=L, seed=99, step=4, S=S)
    for j in range(d):
        lo, hi, p = bracket(x[j], levels, s, L, S)
        vals = np.unique(np.abs(codes[:, j]))
        # mean of |decoded| in units of S
        if levels == UNIFORM:
            mean = np.abs(codes[:, j]).mean() / s
        else:
            k = np.abs(codes[:, j]).astype(np.float64)
            mean = np.where(k == 0, 0.0, 2.0 ** (k - L)).mean()
        target = float(abs(Fraction(float(x[j]))) / Fraction(float(S)))
        sigma = float(hi - lo) * math.sqrt(float(p * (1 - p)) / N)
        slack = 4 * sigma + float(hi - lo) * 2.0 ** -22 + target * 2.0 ** -22
        assert abs(mean - target) <= slack, (j, mean, target, sigma, vals)
        assert len(vals) <= 2


# ------------------------------------------------------------------ T2 variance
@pytest.mark.parametrize("s", [1, 4, 15])
def test_uniform_variance_closed_form_and_qsgd_bound(oracle, s):
    d, N = 16, 1 << 18
    x = synthetic.numpy_normal(1, d, 20)[0]
    S = np.float32(np.linalg.norm(x.astype(np.float64)))
    exact = 0.0
    for j in range(d):
        lo, hi, p = bracket(x[j], UNIFORM, s, 8, S)
        exact += float(S) ** 2 * float((hi - lo) ** 2 * p * (1 - p))
    norm2 = float(np.dot(x.astype(np.float64), x.astype(np.float64)))
    bound = min(d / s ** 2, math.sqrt(d) / s) * norm2
    assert exact <= bound * (1 + 1e-9)
    codes = oracle.quantize(replicas(x, N), s=s, seed=5, step=0, S=S)
    q = codes.astype(np.float64) * (float(S) / s)
    err = ((q - x.astype(np.float64)) ** 2).sum(axis=1)
    mc, se = err.mean(), err.std() / math.sqrt(N)
    assert abs(mc - exact) <= 4 * se + 1e-6 * exact, (mc, exact, se)


# ------------------------------------------------------------ T3 range and sign
@pytest.mark.parametrize("levels,s,L", [(UNIFORM, 15, 8), (UNIFORM, 127, 8), (EXP, 15, 8),
                                        (EXP, 15, 1), (EXP, 15, 15)])
def test_code_range_and_sign(oracle, levels, s, L):
    rng = np.random.default_rng(30)
    W, d = 6, 4096
    g = (rng.standard_t(2, size=(W, d)) * 10.0 ** rng.uniform(-30, 3, size=(W, d))
         ).astype(np.float32)
    g[0, :8] = [0.0, -0.0, 1e-45, -1e-45, 3e38, -3e38, 1.0, -1.0]
    S, _ = oracle.global_scale(g, None, oracle.SCALE_MAXABS)
    codes = oracle.quantize(g, levels=levels, s=s, L=L, seed=1, step=2, S=S)
    top = s if levels == UNIFORM else L
    assert np.abs(codes).max() <= top
    nz = codes != 0
    assert np.all(np.sign(codes[nz]) == np.sign(g[nz]))
    assert codes[0, 0] == 0 and codes[0, 1] == 0


# ----------------------------------------------------------------- T4 on-level inputs
def test_uniform_inputs_on_levels_are_deterministic(oracle):
    s = 15
    S = np.float32(15 * 2.0 ** -3)          # a = s/S = 8 exactly
    k = np.arange(-15, 16)
    x = (k * 2.0 ** -3).astype(np.float32)  # |x| * a = |k| exactly
    for seed, step in [(0, 0), (1, 7), (0xFFFFFFFFFFFFFFFF, 123456)]:
        codes = oracle.quantize(replicas(x, 64), s=s, seed=seed, step=step, S=S)
        assert np.all(codes == k[None, :])


def test_exp_inputs_on_levels_are_deterministic(oracle):
    L = 8
    S = np.float32(4.0)
    idx = np.arange(0, L + 1)
    mag = np.where(idx == 0, 0.0, 2.0 ** (idx - L)) * 4.0
    x = np.concatenate([mag, -mag[1:]]).astype(np.float32)
    want = np.concatenate([idx, -idx[1:]])
    codes = oracle.quantize(replicas(x, 128), levels=EXP, L=L, seed=3, step=9, S=S)
    assert np.all(codes == want[None, :])


def test_zero_scale_gives_zero_codes(oracle):
    g = np.zeros((3, 77), np.float32)
    r = oracle.step(g, s=15)
    assert r["S"] == 0 and not r["codes"].any() and not r["sum"].any()
    assert not r["out"].any()


# ------------------------------------------------------------ T5 enumeration d=3
@pytest.mark.parametrize("levels", [UNIFORM, EXP])
def test_enumerate_outcomes_d3(oracle, levels):
    s, L = 7, 4
    x = np.array([0.3, -0.055, 0.81], np.float32)
    S = np.float32(1.0)
    br = [bracket(xj, levels, s, L, S) for xj in x]
    outcomes = {}
    total = Fraction(0)
    expect = [Fraction(0)] * 3
    for ups in itertools.product((0, 1), repeat=3):
        prob = Fraction(1)
        for (lo, hi, p), up in zip(br, ups):
            prob *= p if up else 1 - p
        total += prob
        vec = tuple((hi if up else lo) * (1 if xj >= 0 else -1)
                    for (lo, hi, p), up, xj in zip(br, ups, x))
        outcomes[vec] = outcomes.get(vec, 0) + prob
        for j in range(3):
            expect[j] += prob * vec[j]
    assert total == 1
    for j in range(3):
        # the expectation is x (up to the fp32 value of x itself)
        assert expect[j] == Fraction(float(x[j])) / Fraction(float(S))
    N = 1 << 20
    codes = oracle.quantize(replicas(x, N), levels=levels, s=s, L=L, seed=17, step=1, S=S)
    vals = {}
    for c in range(-max(s, L), max(s, L) + 1):
        vals[c] = level_value(c, levels, s, L, S)
    keys, counts = np.unique(codes, axis=0, return_counts=True)
    seen = {}
    for row, cnt in zip(keys, counts):
        vec = tuple(vals[int(c)] for c in row)
        assert vec in outcomes, vec
        seen[vec] = cnt
    for vec, prob in outcomes.items():
        pf = float(prob)
        sigma = math.sqrt(pf * (1 - pf) / N)
        freq = seen.get(vec, 0) / N
        assert abs(freq - pf) <= 4 * sigma + 2.0 ** -20, (vec, freq, pf)


# ------------------------------------------------------- T6 allreduce compatibility
@pytest.mark.parametrize("levels,s,L", [(UNIFORM, 15, 8), (UNIFORM, 127, 8), (EXP, 15, 8),
                                        (EXP, 15, 5)])
def test_decoded_sum_equals_sum_of_decoded(oracle, levels, s, L):
    W, d = 8, 2000
    g = synthetic.numpy_normal(W, d, 40)
    S, _ = oracle.global_scale(g)
    codes = oracle.quantize(g, levels=levels, s=s, L=L, seed=2, step=0, S=S)
    total = oracle.aggregate(codes, levels=levels, L=L)
    unit = (Fraction(1, s) if levels == UNIFORM else Fraction(1, 2 ** (L - 1))) \
        * Fraction(float(S))
    for j in range(0, d, 37):
        lhs = sum(level_value(codes[w, j], levels, s, L, S) for w in range(W))
        assert lhs == total[j] * unit
    # and the integer sum is numpy's sum for uniform codes
    if levels == UNIFORM:
        assert np.array_equal(total, codes.sum(axis=0))


def test_decode_mean_is_the_rounded_mean(oracle):
    W, d, s = 8, 4096, 15
    g = synthetic.numpy_normal(W, d, 41)
    r = oracle.step(g, s=s)
    exact = r["codes"].astype(np.float64).sum(axis=0) * (float(r["S"]) / s) / W
    # two fp32 roundings (the unit S/s, then sum*unit); /W is exact for W = 8
    assert np.all(np.abs(r["out"] - exact) <= 3 * np.spacing(np.abs(exact).astype(np.float32)))


def test_exp_value_map_is_additive(oracle):
    L = 8
    for code in range(-L, L + 1):
        val = oracle.code_value(code, EXP, L)
        want = level_value(code, EXP, 15, L, np.float32(1.0)) * 2 ** (L - 1)
        assert val == want


# --------------------------------------------------------------- error feedback
def test_error_feedback_telescopes(oracle):
    """sum_t Q(v_t) + e_T = sum_t g_t: nothing is lost, only delayed."""
    W, d, s, T = 4, 3000, 7, 6
    e = np.zeros((W, d), np.float32)
    acc_q = np.zeros((W, d), np.float64)
    acc_g = np.zeros((W, d), np.float64)
    bound = 0.0
    for t in range(T):
        g = synthetic.numpy_normal(W, d, 100 + t) * np.float32(0.01)
        r = oracle.step(g, e, s=s, seed=8, step=t, ef=True)
        unit = float(r["S"]) / s
        acc_q += r["codes"].astype(np.float64) * unit
        acc_g += g.astype(np.float64)
        # the new residual is at most one level spacing (uniform levels)
        assert np.abs(r["e"]).max() <= unit * (1 + 1e-6)
        bound += 4 * unit * 2.0 ** -23 + float(np.abs(g).max()) * 2.0 ** -23
        e = r["e"]
    diff = np.abs(acc_q + e.astype(np.float64) - acc_g).max()
    assert diff <= bound, (diff, bound)


def test_error_feedback_residual_definition(oracle):
    W, d = 3, 500
    g = synthetic.numpy_normal(W, d, 50)
    e0 = synthetic.numpy_normal(W, d, 51) * np.float32(0.05)
    for levels in (UNIFORM, EXP):
        r = oracle.step(g, e0, levels=levels, s=15, L=6, ef=True, seed=4, step=3)
        v = (g + e0).astype(np.float64)
        q = np.array([[float(level_value(c, levels, 15, 6, r["S"])) for c in row]
                      for row in r["codes"]])
        # one rounding of the difference plus one of the decoded value
        tol = np.spacing(np.abs(v - q).astype(np.float32)) + np.spacing(np.abs(q).astype(np.float32))
        assert np.all(np.abs(r["e"] - (v - q)) <= tol)


def test_multiplier_is_s_over_S_rounded_down(oracle):
    """a is the largest float with a * S <= s, checked in exact rationals."""
    rng = np.random.default_rng(61)
    for _ in range(3000):
        s = int(rng.integers(1, 32768))
        S = np.float32(10.0 ** rng.uniform(-30, 30))
        a = oracle.uniform_multiplier(s, S)
        up = np.nextafter(a, np.float32(np.inf))
        assert Fraction(float(a)) * Fraction(float(S)) <= s
        assert Fraction(float(up)) * Fraction(float(S)) > s
    assert oracle.uniform_multiplier(15, np.float32(0.0)) == 0
    assert oracle.uniform_multiplier(15, np.float32(np.inf)) == 0


def test_no_level_beyond_s_at_the_scale(oracle):
    """Inputs with |x| = S (a single-coordinate worker) are where a
    round-to-nearest multiplier would overshoot s; the codes stay within s and
    almost always equal +-s."""
    rng = np.random.default_rng(60)
    for s in (15, 127):
        x = rng.uniform(0.5, 2.0, 400000).astype(np.float32)
        r = x * (np.float32(s) / x)
        over = x[r > s][:12]
        assert over.size == 12
        for xv in over:
            for sign in (1, -1):
                codes = oracle.quantize(replicas([sign * xv], 1 << 19), s=s, seed=int(xv * 1e6),
                                        step=1, S=xv)
                assert np.abs(codes).max() <= s
                assert (codes == sign * s).mean() > 0.999


def test_inputs_beyond_the_scale_are_clamped(oracle):
    """A scale below some |x| (not what the global scale produces) clamps the
    code to +-s."""
    x = np.array([2.0, -3.0, 0.5], np.float32)
    codes = oracle.quantize(replicas(x, 256), s=15, seed=2, step=0, S=np.float32(1.0))
    assert np.all(codes[:, 0] == 15) and np.all(codes[:, 1] == -15)
    assert np.all(np.abs(codes[:, 2]) <= 15)


# ------------------------------------------------- the rounding decision, exactly
def _exact_code(r, f):
    """floor(r + f 2^-23) in rationals: the uniform-level code of r = fl(v a)."""
    return math.floor(Fraction(float(r)) + Fraction(int(f), 1 << 23))


def test_uniform_code_is_exact_floor_at_decision_boundaries(oracle):
    """r = v a sitting a fraction of an ulp of (1 - p) away from the decision
    boundary u = 1 - p, on both sides, and r = -u exactly.  With S = s the
    multiplier is exactly 1, so r = v.  A fraction taken with a float
    subtraction, fl(r - floor(r)), rounds 1 - u - 2^-26 to 1 - u and flips
    the first kind to a round-up; the exact rule floor(r + u) does not."""
    s, seed, step = 15, 7, 1
    assert oracle.uniform_multiplier(s, np.float32(s)) == np.float32(1.0)
    js, fs = [], []
    for j in range(4000):
        f = oracle.uniform_bits(seed, 0, step, 0, j)
        if (1 << 20) <= f < (1 << 21):  # u in [1/8, 1/4): |r| has ulp 2^-26
            js.append(j)
            fs.append(f)
    assert len(js) >= 200
    js, fs = np.array(js[:240], np.int64), np.array(fs[:240], np.int64)
    u = fs.astype(np.float64) / (1 << 23)
    kinds = np.arange(js.size) % 3
    r = np.where(kinds == 0, -(u + 2.0 ** -26),           # just past the boundary: -1
                 np.where(kinds == 1, -(u - 2.0 ** -26),  # just short of it: 0
                          -u))                             # on it: 0
    v = r.astype(np.float32)
    assert np.array_equal(v.astype(np.float64), r)  # all exactly representable
    codes = oracle.quantize(v[None, :], s=s, seed=seed, step=step, S=np.float32(s), js=js)[0]
    want = np.array([_exact_code(x, f) for x, f in zip(v, fs)])
    assert np.array_equal(want[kinds == 0], -np.ones((kinds == 0).sum()))
    assert not want[kinds != 0].any()
    assert np.array_equal(codes, want)


def test_uniform_code_is_exact_floor_random(oracle):
    """20000 random r of both signs and magnitudes from 2^-40 to s, exact check."""
    s, seed, step = 127, 3, 9
    rng = np.random.default_rng(5)
    n = 20000
    mag = np.exp2(rng.uniform(-40, np.log2(s), n))
    v = (mag * rng.choice([-1.0, 1.0], n)).astype(np.float32)
    js = np.arange(n, dtype=np.int64) * 7 + 11
    codes = oracle.quantize(v[None, :], s=s, seed=seed, step=step, S=np.float32(s), js=js)[0]
    fs = [oracle.uniform_bits(seed, 0, step, 0, int(j)) for j in js]
    want = np.array([_exact_code(x, f) for x, f in zip(v, fs)])
    assert np.array_equal(codes, want)
