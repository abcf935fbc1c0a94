"""The fused pass rounds exponential levels by an exponent carry: r = fl(v a)
is scaled by 2^(L-127) rounding toward zero, which puts the finest level on
2^-126 and the bottom bracket in the subnormal range; the 23 random bits are
added to the bit pattern and the result masked to sign and exponent.  The
exponent field is then the level index, and a 512-entry table maps the top
nine bits to the signed code.

This file emulates that bit arithmetic on the host (numpy, exact) and checks
it against the oracle's exponential quantizer (NUQSGD's nonuniform levels,
rounded up with probability (r - lo)/(hi - lo)) on inputs that reach every
bracket: zeros of both signs, subnormal inputs, inputs exactly on a level,
the maximum, and values spread over nine decades.  It pins the derivation
the kernel relies on, independently of the GPU."""
import numpy as np
import pytest


def emulate(g, a, L, f):
    """Codes and level values (in finest-level units) of the exponent carry."""
    r = (g.astype(np.float32) * np.float32(a)).astype(np.float32)   # fl(v a), round to nearest
    x = r.astype(np.float64) * 2.0 ** (L - 127)                      # exact in double
    tiny = 2.0 ** -149
    sub = np.abs(x) < 2.0 ** -126
    xs = np.where(sub, np.trunc(x / tiny) * tiny, x)                 # toward zero, fp32 grid
    rs = xs.astype(np.float32)
    assert np.array_equal(rs.astype(np.float64), xs)
    y = ((rs.view(np.uint32).astype(np.uint64) + f.astype(np.uint64)) & 0xFFFFFFFF)
    y = y.astype(np.uint32)
    level = (y & np.uint32(0xFF800000)).view(np.float32)
    h = (y >> 23).astype(np.int64)                                   # sign, exponent field
    e = h & 255
    idx = np.where(e <= L, e, 0)
    code = np.where(h >> 8, -idx, idx)
    return code, level.astype(np.float64) * 2.0 ** 126


@pytest.mark.parametrize("L", [1, 2, 3, 5, 8, 12, 15])
def test_exponent_carry_equals_the_oracle(oracle, L):
    rng = np.random.default_rng(L)
    W, n = 3, 6000
    g = (rng.standard_normal((W, n)) * 10.0 ** rng.uniform(-9, 0, (W, n))).astype(np.float32)
    fin = 2.0 ** -(L - 1)
    g[0, :10] = [0.0, -0.0, 1e-40, -1e-40, 1.0, -1.0, fin, -fin, fin / 2, -3 * fin / 4]
    S = np.float32(np.abs(g).max())
    a = oracle.uniform_multiplier(1, S)  # 1/S rounded toward zero, as the kernel's
    step, seed = 3, 7
    ref = oracle.quantize(g, levels=1, L=L, seed=seed, step=step, S=S)
    f = np.array([[oracle.uniform_bits(seed, 0, step, w, j) for j in range(n)]
                  for w in range(W)], dtype=np.uint32)
    code, units = emulate(g, a, L, f)
    assert np.array_equal(code, ref)
    # the level value is 2^(idx-1) finest-level units, the sum's summand
    want = np.vectorize(lambda c: oracle.code_value(int(c), 1, L))(ref)
    assert np.array_equal(units, want.astype(np.float64))
    # summing the levels as fp32 over the workers is exact
    fsum = (units * 2.0 ** -126).astype(np.float32).sum(axis=0, dtype=np.float32)
    assert np.array_equal(fsum.astype(np.float64) * 2.0 ** 126, want.sum(axis=0))


def test_table_covers_every_top_nine_bits():
    """Any 32-bit pattern's top nine bits index the 512-entry table."""
    y = np.array([0, 0x007FFFFF, 0x7F800000, 0x7FFFFFFF, 0x80000000, 0xFFFFFFFF], np.uint64)
    assert ((y >> 23) < 512).all()
