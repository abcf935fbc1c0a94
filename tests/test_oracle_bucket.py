"""Pins of the oracle's per-bucket composition (``oracle.step_bucketed``).

Per bucket of consecutive coordinates, the path is the global-scale path of
"Quantize Once, Train Fast: Allreduce-Compatible Compression with Provable
Guarantees" (Abstract: global norm scaling) restricted to the bucket.  The
composition adds no arithmetic, so what can go wrong is the plumbing: a wrong
slice, a wrong coordinate index for the uniforms, a scale taken from the wrong
bucket or worker, a decode with the wrong bucket's unit.  Each test below
fails on one of those:

* one bucket covering all of d is the unbucketed path, bit for bit;
* each S_k is the fp64 norm (or max-abs) of its slice, recomputed in numpy;
* the codes of bucket k are the full-row quantizer's codes at those columns
  with S = S_k (the uniforms follow the global coordinate index);
* a zero bucket stays zero while its neighbours do not (no scale leaks);
* Monte Carlo: the decoded mean is unbiased per coordinate and its variance
  is the stochastic-rounding closed form with each bucket's own unit.
"""
import numpy as np
import pytest

import synthetic


def _g(W, d, seed, lo=-4, hi=0, seg=100):
    return synthetic.make_gradients(W, d, "student_t3", seed=seed, seg=seg, lo=lo,
                                    hi=hi).numpy()


@pytest.mark.parametrize("levels,kw", [(0, dict(s=15)), (1, dict(L=8))])
@pytest.mark.parametrize("ef", [False, True])
def test_one_bucket_is_the_global_step(oracle, levels, kw, ef):
    W, d = 3, 1000
    g = _g(W, d, 1)
    e = _g(W, d, 2, lo=-6, hi=-3) if ef else None
    a = oracle.step(g, e, levels=levels, seed=5, step=2, ef=ef, bits=5, **kw)
    b = oracle.step_bucketed(g, e, bucket=1024, levels=levels, seed=5, step=2, ef=ef, bits=5,
                             **kw)
    assert b["S"].shape == (1,) and b["S"][0] == a["S"]
    for key in ("codes", "packed", "sum"):
        assert np.array_equal(a[key], b[key]), key
    assert np.array_equal(a["out"].view(np.uint32), b["out"].view(np.uint32))
    if ef:
        assert np.array_equal(a["e"].view(np.uint32), b["e"].view(np.uint32))


@pytest.mark.parametrize("scale_kind", [0, 1])
def test_bucket_scales_are_slice_norms(oracle, scale_kind):
    W, d, B = 4, 1000, 128  # ragged last bucket of 104
    g = _g(W, d, 3, seg=50)
    e = _g(W, d, 4, lo=-6, hi=-2)
    r = oracle.step_bucketed(g, e, bucket=B, scale_kind=scale_kind, ef=True, bits=5)
    v = (g + e).astype(np.float32)  # v = fl(g + e)
    assert r["S"].shape == (-(-d // B),)
    for k in range(r["S"].shape[0]):
        sl = v[:, k * B:(k + 1) * B].astype(np.float64)
        if scale_kind == 0:
            want = np.sqrt((sl * sl).sum(axis=1)).max()
            assert abs(float(r["S"][k]) - want) <= 1e-6 * want
        else:
            assert r["S"][k] == np.float32(np.abs(sl).max())


def test_bucket_codes_follow_global_coordinates(oracle):
    W, d, B = 2, 700, 128
    g = _g(W, d, 5)
    r = oracle.step_bucketed(g, bucket=B, s=7, seed=11, step=3, bits=4)
    for k in range(r["S"].shape[0]):
        full = oracle.quantize(g, s=7, seed=11, step=3, S=r["S"][k])
        cols = slice(k * B, (k + 1) * B)
        assert np.array_equal(r["codes"][:, cols], full[:, cols]), k


def test_zero_bucket_stays_zero(oracle):
    W, d, B = 2, 512, 128
    g = _g(W, d, 6)
    g[:, 128:256] = 0.0
    r = oracle.step_bucketed(g, bucket=B, s=15, bits=5)
    assert r["S"][1] == 0.0 and (r["S"][[0, 2, 3]] > 0).all()
    assert not r["codes"][:, 128:256].any() and not r["out"][128:256].any()
    assert r["codes"][:, :128].any() and r["codes"][:, 256:].any()


def test_small_bucket_keeps_small_coordinates(oracle):
    """A bucket of small entries next to a bucket of large ones: with one global
    (max-abs) scale the small entries round to 0 or the first level; with their
    own bucket scale they use the whole level range."""
    W, d, B, s = 1, 256, 128, 15
    rng = np.random.default_rng(0)
    g = np.concatenate([rng.uniform(-1e-3, 1e-3, 128), rng.uniform(-1, 1, 128)])
    g = g.astype(np.float32)[None, :]
    glob = oracle.step(g, s=s, bits=5, scale_kind=1)
    buck = oracle.step_bucketed(g, bucket=B, s=s, bits=5, scale_kind=1)
    assert np.abs(glob["codes"][:, :128]).max() <= 1
    # max-abs scale: the bucket's largest entry sits exactly on the top level
    assert np.abs(buck["codes"][:, :128]).max() == s


@pytest.mark.parametrize("levels,kw", [(0, dict(s=3)), (1, dict(L=4))])
def test_bucketed_mean_unbiased_with_closed_form_variance(oracle, levels, kw):
    W, d, B, n = 2, 8, 4, 3000
    rng = np.random.default_rng(1)
    g = np.concatenate([rng.uniform(-1e-2, 1e-2, (W, 4)), rng.uniform(-3, 3, (W, 4))], axis=1)
    g = g.astype(np.float32)
    outs = np.empty((n, d))
    S = None
    for t in range(n):
        r = oracle.step_bucketed(g, bucket=B, levels=levels, seed=t, step=t, bits=5, **kw)
        outs[t] = r["out"]
        S = r["S"]
    vbar = g.astype(np.float64).mean(axis=0)
    # closed form per coordinate: (1/W^2) sum_w (hi - lo)^2 p (1 - p), with lo, hi
    # the bracketing levels of |v| on bucket k's grid and p its rounding-up chance
    var = np.zeros(d)
    for j in range(d):
        Sk = float(S[j // B])
        for w in range(W):
            x = abs(float(g[w, j])) / Sk
            if levels == 0:
                lo = np.floor(x * kw["s"]) / kw["s"]
                hi = lo + 1.0 / kw["s"]
            else:
                lv = [0.0] + [2.0 ** -(kw["L"] - 1 - i) for i in range(kw["L"])]
                i = max(i for i in range(len(lv)) if lv[i] <= x)
                lo, hi = lv[i], lv[min(i + 1, len(lv) - 1)]
            p = 0.0 if hi == lo else (x - lo) / (hi - lo)
            var[j] += (Sk * (hi - lo)) ** 2 * p * (1 - p) / W ** 2
    mean = outs.mean(axis=0)
    assert (np.abs(mean - vbar) <= 5 * np.sqrt(var / n) + 1e-6).all()
    emp = ((outs - vbar) ** 2).mean(axis=0).sum()
    assert abs(emp - var.sum()) <= 0.1 * var.sum()
