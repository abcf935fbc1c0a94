"""Pins for the oracle's Philox-4x32-10 and its uniform draws.

Philox-4x32-10 (Salmon et al., SC'11) is also what cuRAND's host generator
CURAND_RNG_PSEUDO_PHILOX4_32_10 computes.  That generator runs on the CPU, so
the oracle's Philox is compared with it as a library routine: with the
generator seeded by a 64-bit seed and offset by 4 * 65536 * k outputs, its
output block g (for g < 65536) is Philox(ctr = (lo32 k, hi32 k, g, 0),
key = (lo32 seed, hi32 seed)).  That covers both key words and counter words
0, 1 and 2; the draws below keep counter word 3 at zero for every d < 2^34.
"""
import ctypes
import ctypes.util
import os

import numpy as np
import pytest

CURAND_RNG_PSEUDO_PHILOX4_32_10 = 161


def _curand():
    for cand in ("/usr/local/cuda/lib64/libcurand.so", ctypes.util.find_library("curand")):
        if cand and (os.path.exists(cand) or not cand.startswith("/")):
            try:
                return ctypes.CDLL(cand)
            except OSError:
                continue
    return None


def curand_host_words(lib, seed, n, offset):
    gen = ctypes.c_void_p()
    assert lib.curandCreateGeneratorHost(ctypes.byref(gen), CURAND_RNG_PSEUDO_PHILOX4_32_10) == 0
    try:
        assert lib.curandSetPseudoRandomGeneratorSeed(gen, ctypes.c_ulonglong(seed)) == 0
        assert lib.curandSetGeneratorOffset(gen, ctypes.c_ulonglong(offset)) == 0
        buf = (ctypes.c_uint32 * n)()
        assert lib.curandGenerate(gen, buf, ctypes.c_size_t(n)) == 0
        return np.frombuffer(buf, dtype=np.uint32).copy()
    finally:
        lib.curandDestroyGenerator(gen)


SEEDS = [0, 0x0123456789ABCDEF, 0xFFFFFFFFFFFFFFFF, 0x51D5EED, 0x9E3779B97F4A7C15]
BLOCKS = [0, 1, 7, (1 << 32) + 5, (3 << 32) + 0xABCDE, 0xFFFFFFFF, (1 << 42) - 1]


@pytest.mark.parametrize("seed", SEEDS)
def test_philox_equals_curand_host_generator(oracle, seed):
    lib = _curand()
    if lib is None:
        pytest.skip("libcurand not loadable on this host")
    G = 48
    for k in BLOCKS:
        words = curand_host_words(lib, seed, 4 * G, 4 * 65536 * k)
        for g in range(G):
            ctr = [k & 0xFFFFFFFF, (k >> 32) & 0xFFFFFFFF, g, 0]
            got = oracle.philox4x32(ctr, (seed & 0xFFFFFFFF, seed >> 32))
            assert list(got) == list(words[4 * g:4 * g + 4]), (hex(seed), k, g)


def test_philox_round_count_matters(oracle):
    # fewer rounds give different blocks; 10 is the member the path uses
    a = oracle.philox4x32([1, 2, 3, 4], (5, 6), 10)
    b = oracle.philox4x32([1, 2, 3, 4], (5, 6), 7)
    assert list(a) != list(b)


def test_uniform_bits_follow_the_counter_layout(oracle):
    # coordinate j of worker w at step t uses block (j>>2) of the stream keyed by
    # (seed, tag), word j & 3, top 23 bits; counter word 3 carries j >> 34.
    seed, tag = 0x0123456789ABCDEF, 0x4C510003
    rng = np.random.default_rng(3)
    for _ in range(200):
        j = int(rng.integers(0, 1 << 40))
        w = int(rng.integers(0, 64))
        t = int(rng.integers(0, 1 << 31))
        q = j >> 2
        blk = oracle.philox4x32([q & 0xFFFFFFFF, t, w, q >> 32],
                                (seed & 0xFFFFFFFF, (seed >> 32) ^ tag))
        assert oracle.uniform_bits(seed, tag, t, w, j) == int(blk[j & 3]) >> 9


def test_uniform_bits_are_uniform(oracle):
    # chi-square over 64 equal bins of u = f / 2^23 for 2^16 consecutive coordinates
    n, bins = 1 << 16, 64
    f = np.array([oracle.uniform_bits(7, 0, 3, 1, j) for j in range(n)], dtype=np.uint32)
    assert f.max() < (1 << 23)
    counts = np.bincount(f >> (23 - 6), minlength=bins)
    exp = n / bins
    chi2 = float(((counts - exp) ** 2 / exp).sum())
    # 63 degrees of freedom: P(chi2 > 110) < 2e-4
    assert chi2 < 110.0, chi2


def test_streams_differ_by_worker_step_and_tag(oracle):
    base = [oracle.uniform_bits(11, 0, 0, 0, j) for j in range(64)]
    for kw in (dict(tag=0, step=1, worker=0), dict(tag=0, step=0, worker=1),
               dict(tag=0x4C510000, step=0, worker=0)):
        other = [oracle.uniform_bits(11, kw["tag"], kw["step"], kw["worker"], j)
                 for j in range(64)]
        assert sum(a == b for a, b in zip(base, other)) <= 1
