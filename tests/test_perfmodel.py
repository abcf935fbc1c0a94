"""The bandwidth model (host arithmetic only)."""
import math

import numpy as np
import pytest

from allreduce_compatible_gradient_global_b200 import perfmodel as pm


def test_fit_recovers_launch_and_bandwidth():
    rng = np.random.default_rng(0)
    sizes = np.array([1e6, 4e6, 1.6e7, 6.4e7, 2.6e8, 1e9])
    t = 7e-6 + sizes / 5.5e12
    launch, bw = pm.fit_launch_and_bandwidth(sizes, t)
    assert abs(launch - 7e-6) < 1e-12 and abs(bw - 5.5e12) / 5.5e12 < 1e-9
    noisy = t * (1 + 1e-3 * rng.standard_normal(t.size))
    launch, bw = pm.fit_launch_and_bandwidth(sizes, noisy)
    assert abs(bw - 5.5e12) / 5.5e12 < 0.01
    with pytest.raises(ValueError):
        pm.fit_launch_and_bandwidth([5, 5], [1, 2])


def test_step_bytes_of_the_resnet50_sized_workload():
    W, d = 8, 25_557_032
    p1, p2 = pm.step_bytes(W, d, bits=5, sum_bytes=1)
    assert p1 == 4 * W * d
    assert p2 == 1_073_395_784  # read g, 5-bit padded rows, int8 sum, fp32 mean
    q1, q2 = pm.step_bytes(W, d, bits=5, sum_bytes=1, ef=True)
    assert q1 == 2 * p1 and q2 == p2 + 8 * W * d


def test_ring_allreduce_cost():
    assert pm.ring_allreduce_seconds(1e9, 1, 770e9, 1e-5) == 0.0
    t2 = pm.ring_allreduce_seconds(1e9, 2, 770e9, 1e-5)
    t8 = pm.ring_allreduce_seconds(1e9, 8, 770e9, 1e-5)
    assert math.isclose(t2, 1e-5 + 1e9 / 770e9)
    assert math.isclose(t8, 1e-5 + 1.75e9 / 770e9)


def test_crossover_separates_the_regimes():
    m = pm.Machine()
    for ranks in (2, 4, 8):
        d0 = pm.crossover_d(ranks, bits=5, sum_bytes=1, m=m)
        assert d0 is not None and d0 > 1
        for d in (d0, 2 * d0, 100 * d0):
            assert pm.dp_step_seconds(d, ranks, 5, 1, m) < pm.dp_step_seconds(
                d, ranks, 5, 1, m, compressed=False)
        assert pm.dp_step_seconds(d0 - 1, ranks, 5, 1, m) >= pm.dp_step_seconds(
            d0 - 1, ranks, 5, 1, m, compressed=False)
    # a single GPU has no exchange: compression never pays
    assert pm.crossover_d(1, m=m) is None


def test_large_d_ratio_follows_the_byte_counts():
    m = pm.Machine()
    d, n = 1 << 40, 8
    fast = pm.dp_step_seconds(d, n, 5, 1, m)
    slow = pm.dp_step_seconds(d, n, 5, 1, m, compressed=False)
    per_coord_fast = (4 / m.hbm + (4 + 5 / 8) / (m.hbm * m.pass2_efficiency) + 5 / m.hbm
                      + 2 * (n - 1) / n / m.link)
    per_coord_slow = 2 * (n - 1) / n * 4 / m.link
    assert math.isclose(slow / fast, per_coord_slow / per_coord_fast, rel_tol=1e-3)


def test_chunked_pipeline_model():
    """One chunk is the unpipelined step.  Pipelining hides the shorter stage
    but each chunk pays a launch and an all-reduce latency again: with 15 us
    per all-reduce it loses at 25.6 M coordinates and wins at 2^30, never
    beating the slower stage over all of d."""
    from allreduce_compatible_gradient_global_b200 import perfmodel as pm
    m = pm.Machine()
    N = 8

    def parts(d):
        norm = m.launch + 4.0 * d / m.hbm
        scale = pm.ring_allreduce_seconds(4.0, N, m.link, m.allreduce_alpha)
        quant = m.launch + 5.0 * d / (m.hbm * m.pass2_efficiency)
        summ = pm.ring_allreduce_seconds(float(d), N, m.link, m.allreduce_alpha)
        decode = m.launch + 5.0 * d / m.hbm
        return norm, scale, quant, summ, decode

    d = 25_557_032
    norm, scale, quant, summ, decode = parts(d)
    one = pm.dp_step_seconds(d, N, m=m, chunks=1)
    assert abs(one - (norm + scale + quant + summ + decode)) < 1e-12
    assert pm.dp_step_seconds(d, N, m=m, chunks=4) > one
    d = 1 << 30
    norm, scale, quant, summ, decode = parts(d)
    one = pm.dp_step_seconds(d, N, m=m, chunks=1)
    four = pm.dp_step_seconds(d, N, m=m, chunks=4)
    assert four < one
    assert four > norm + scale + decode + max(quant, summ)
    assert pm.dp_step_seconds(d, N, m=m, chunks=1 << 16) > four


def test_natural_exchange_link_bytes():
    """Sharded: (N-1)/N * 2n (all-to-all of codes) + (N-1)/N * 4n (all-gather of
    fp32 shard sums) = 3/4 of a ring fp32 all-reduce's 2 (N-1)/N * 4n; gather:
    (N-1) * 2n.  Checked with free HBM and latencies so only link time is left."""
    m = pm.Machine(hbm=float("inf"), allreduce_alpha=0.0, launch=0.0)
    n = 8 * 1_000_000
    for N in (2, 4, 8):
        fp32 = pm.dp_step_seconds(n, N, m=m, compressed=False)
        sharded = pm.nat_step_seconds(n, N, m=m, sharded=True)
        gather = pm.nat_step_seconds(n, N, m=m)
        assert sharded == pytest.approx(0.75 * fp32, rel=1e-12)
        assert gather == pytest.approx((N - 1) * 2 * n / m.link, rel=1e-12)


def test_natural_exchange_on_one_rank_is_the_two_kernels():
    m = pm.Machine()
    n = 1 << 24
    want = (m.launch + 6.0 * n / (m.hbm * 0.77)) + (m.launch + 6.0 * n / (m.hbm * 0.91))
    assert pm.nat_step_seconds(n, 1, m=m) == pytest.approx(want)
    assert pm.nat_step_seconds(n, 1, m=m, sharded=True) == pytest.approx(want)


def test_allreduce_compatible_exchange_beats_natural_compression():
    """Bandwidth regime (d >= 2^25): the integer all-reduce of the shared-scale
    codes beats both natural-compression exchanges at every rank count, and the
    sharded form beats the gather from 4 ranks on.  Latency regime (d = 2^20,
    2 and 4 ranks; at 8 ranks the three are within 0.2 us): the integer exchange
    pays two collectives (the scale's MAX and the sum), the natural gather one,
    and the gather is the fastest of the three."""
    for N in (2, 4, 8):
        for d in (1 << 25, 1 << 30):
            int8 = pm.dp_step_seconds(d, N)
            assert int8 < pm.nat_step_seconds(d, N, sharded=True)
            assert int8 < pm.nat_step_seconds(d, N)
            if N >= 4:
                assert pm.nat_step_seconds(d, N, sharded=True) < pm.nat_step_seconds(d, N)
    for N in (2, 4):
        d = 1 << 20
        gather = pm.nat_step_seconds(d, N)
        assert gather < pm.dp_step_seconds(d, N)
        assert gather < pm.nat_step_seconds(d, N, sharded=True)


def test_natural_exchange_crossover_against_fp32():
    """Sharded natural compression overtakes the fp32 all-reduce only at large n
    (about 92 M coordinates on 4 ranks and 35 M on 8 with the default machine),
    never on 2 ranks; the gather form never does from 4 ranks on."""
    assert pm.nat_crossover_d(2) is None
    c4, c8 = pm.nat_crossover_d(4), pm.nat_crossover_d(8)
    assert 85e6 < c4 < 100e6 and 30e6 < c8 < 40e6
    for N in (4, 8):
        c = pm.nat_crossover_d(N)
        assert pm.nat_step_seconds(c, N, sharded=True) < pm.dp_step_seconds(c, N, compressed=False)
        assert pm.nat_step_seconds(c - 1, N, sharded=True) >= \
            pm.dp_step_seconds(c - 1, N, compressed=False)
        assert pm.nat_crossover_d(N, sharded=False) is None

