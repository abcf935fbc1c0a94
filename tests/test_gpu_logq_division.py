"""The log quantizer divides every entry by its matrix's max and every log by
log1p(alpha) with the divisor's reciprocal and one fused correction
(Markstein's method), falling back to IEEE division where the reciprocal,
the remainder or the correction could underflow.  Its codes are then those of
IEEE division, which the oracle uses; this test checks the division itself,
through gq_selftest_fma_div (the kernel's own helper), bit for bit against
torch's IEEE fp32 division on the GPU, over divisors spread across the
exponent range, edge mantissas, the extremes and log1p(10), with dividends
drawn across [0, b] by exponent (so the domain's boundary and the fallback
below it are both exercised)."""
import math

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import allreduce_compatible_gradient_global_b200 as gq
    return gq


def f32(bits):
    return float(np.array([bits], dtype=np.uint32).view(np.float32)[0])


def divisors():
    rng = np.random.default_rng(11)
    out = [f32(b) for b in (0x3F800000, 0x3F7FFFFF, 0x3F800001, 0x3FFFFFFF, 0x3FC00000,
                            0x3FAAAAAB, 0x3F000001, 0x40866666, 0x00800000, 0x00FFFFFF,
                            0x7F7FFFFF, 0x7F000000, 0x3F7FFFFE, 0x0D7FFFFF, 0x7E7FFFFF,
                            0x0000FFFF)]
    out.append(float(np.float32(math.log1p(10.0))))
    for e in rng.integers(-125, 126, size=47):
        out.append(float(np.float32(math.ldexp(1.0 + rng.random(), int(e)))))
    return out


def dividends(b, n, rng):
    """[0, b]: exponent uniform over the 150 binades below b's, mantissa random,
    plus 0, b and b's neighbours below."""
    eb = math.frexp(b)[1]
    e = rng.integers(eb - 150, eb + 1, size=n)
    m = rng.random(n)
    a = np.ldexp(0.5 + 0.5 * m, e).astype(np.float32)
    a = np.minimum(a, np.float32(b))
    a[:3] = [0.0, b, np.nextafter(np.float32(b), np.float32(0))]
    a[3:64:7] = 0.0  # zeros among the others: exact on either road
    return a


def test_division_matches_ieee_bit_for_bit(gq):
    rng = np.random.default_rng(5)
    n = 1 << 20
    for b in divisors():
        a = torch.from_numpy(dividends(b, n, rng)).cuda()
        got = torch.empty_like(a)
        gq.gq_selftest_fma_div(a, b, got)
        want = a / torch.tensor(b, dtype=torch.float32, device="cuda")
        torch.cuda.synchronize()
        bad = (got.view(torch.int32) != want.view(torch.int32)).nonzero()
        assert bad.numel() == 0, (b, a[bad[:4, 0]].tolist(), got[bad[:4, 0]].tolist(),
                                  want[bad[:4, 0]].tolist())
