"""The threaded CPU figure of bench.py runs the oracle's own routines by worker
rows (the scale), then by coordinate chunks (codes, packing, sums, means, error
feedback).  Its result must equal the oracle's one-call step bit for bit, or the
figure would be timing a different computation."""
import os
import sys

import numpy as np
import pytest

import synthetic

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("levels,s,L,scale_kind,bits,W,d,threads,ef", [
    (0, 15, 8, 0, 5, 3, 5037, 3, False),      # ragged last chunk and block
    (1, 15, 8, 1, 5, 4, 20001, 5, False),     # exponential levels, max-abs scale
    (0, 127, 8, 0, 8, 2, 1000, 8, False),     # more threads than chunks need
    (0, 7, 8, 0, 4, 8, 129, 2, False),        # one block and a single coordinate over
    (0, 127, 8, 0, 8, 8, 3000, 4, True),      # the d = 2^30 settings, error feedback
    (1, 15, 6, 0, 5, 3, 777, 3, True),        # exponential levels with error feedback
])
def test_threaded_oracle_step_equals_the_oracle_step(oracle, levels, s, L, scale_kind, bits,
                                                     W, d, threads, ef):
    sys.path.insert(0, ROOT)
    import bench
    g = synthetic.make_gradients(W, d, "student_t3", seed=d, seg=100, lo=-3, hi=0).numpy()
    e = (synthetic.make_gradients(W, d, "normal", seed=d + 1).numpy() * 1e-2) if ef else None
    ref = oracle.step(g, e, levels=levels, s=s, L=L, scale_kind=scale_kind, seed=7, bits=bits,
                      ef=ef)
    got = bench.oracle_step_threaded(g, threads, e, levels=levels, s=s, L=L,
                                     scale_kind=scale_kind, bits=bits, seed=7)
    assert got["S"] == ref["S"]
    assert np.array_equal(got["packed"], ref["packed"])
    assert np.array_equal(got["sum"], ref["sum"])
    assert np.array_equal(got["out"].view(np.uint32), ref["out"].view(np.uint32))
    if ef:
        assert np.array_equal(got["e"].view(np.uint32), ref["e"].view(np.uint32))
    else:
        assert got["e"] is None
