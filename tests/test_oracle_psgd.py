"""Pins of the PowerSGD + log-quantizer oracle (``oracle.psgd``).

What the mathematics fixes, checked without re-typing the oracle's steps:

* Modified Gram-Schmidt returns orthonormal columns spanning the same
  nested subspaces: P_hat^T P_hat = I and R = P_hat^T P is upper triangular
  with a positive diagonal (P = P_hat R is the thin QR factorization, unique
  for full column rank), checked against numpy's QR up to column signs.
* Exact recovery: with the quantizer replaced by the identity, one step on
  worker gradients G_w = A B_w^T that share a rank-r column space returns
  Ghat = mean_w G_w (power iteration from a generic Q finds the column space;
  P_hat P_hat^T then projects onto it).  A transposed operand, a sum in place of
  the mean of Q, or a P_hat from the wrong columns fails this.
* Error feedback telescopes (LQ-SGD review, "What carries the argument":
  E_t = G'_t - Ghat_t is added back): over T steps with the log quantizer on,
  sum_t mean_w G_t = sum_t Ghat_t + mean_w E_T.
* The deferred error: E of step t+1 is M_t - Ghat_t, from the state alone.
* The log quantizer is wired in: Ghat stays close to the unquantized one, the
  factor codes are those of ``oracle.logq_quantize`` with steps 2t and 2t+1.
"""
import numpy as np
import pytest


@pytest.fixture(scope="module")
def psgd(oracle):
    from oracle import psgd
    return psgd


def test_mgs_is_thin_qr(psgd):
    rng = np.random.default_rng(0)
    for n, r in ((50, 1), (64, 4), (300, 7), (9, 8)):
        P = rng.standard_normal((n, r))
        Ph = psgd.mgs(P)
        assert np.allclose(Ph.T @ Ph, np.eye(r), atol=1e-12)
        R = Ph.T @ P
        assert np.allclose(np.tril(R, -1), 0, atol=1e-12)
        assert (np.diag(R) > 0).all()
        Qn, Rn = np.linalg.qr(P)
        sgn = np.sign(np.diag(Rn))
        assert np.allclose(Ph, Qn * sgn, atol=1e-10)


def test_mgs_zero_column_stays_zero(psgd):
    rng = np.random.default_rng(1)
    P = rng.standard_normal((40, 3))
    P[:, 1] = 0.0
    Ph = psgd.mgs(P)
    assert np.allclose(Ph[:, 1], 0, atol=1e-12)
    assert np.isclose(np.linalg.norm(Ph[:, 0]), 1) and np.isclose(np.linalg.norm(Ph[:, 2]), 1)
    assert abs(Ph[:, 0] @ Ph[:, 2]) < 1e-12


def _lowrank_workers(rng, W, shapes, r):
    mats = []
    for n, m in shapes:
        A = rng.standard_normal((n, r))
        mats.append(np.stack([A @ rng.standard_normal((m, r)).T for _ in range(W)]))
    return np.concatenate([x.reshape(W, -1) for x in mats], axis=1)


@pytest.mark.parametrize("r", [1, 3, 8])
def test_exact_recovery_without_quantization(psgd, r):
    rng = np.random.default_rng(r)
    W, shapes = 3, [(40, 30), (17, 64)]
    G = _lowrank_workers(rng, W, shapes, r)
    Q0 = rng.standard_normal(sum(m * r for _, m in shapes))
    out = psgd.lqsgd_step(G, np.zeros_like(G), np.zeros(sum(n * r for n, _ in shapes)), Q0,
                          shapes=shapes, rank=r, have_prev=False, lq=False)
    assert np.allclose(out["Ghat"], G.mean(axis=0), rtol=0, atol=1e-9 * np.abs(G).max())
    # the error left is zero, and the next step sees it through the state
    assert np.allclose(out["E_next"], G - out["Ghat"][None], atol=1e-12 * np.abs(G).max())


def test_error_feedback_telescopes(psgd):
    rng = np.random.default_rng(7)
    W, r, shapes, T = 4, 2, [(32, 24), (16, 40)], 6
    dim = sum(n * m for n, m in shapes)
    M = np.zeros((W, dim))
    P = np.zeros(sum(n * r for n, _ in shapes))
    Q = rng.standard_normal(sum(m * r for _, m in shapes))
    sum_g = np.zeros(dim)
    sum_ghat = np.zeros(dim)
    for t in range(T):
        G = rng.standard_normal((W, dim))
        out = psgd.lqsgd_step(G, M, P, Q, shapes=shapes, rank=r, have_prev=t > 0, seed=3,
                              step=t)
        sum_g += G.mean(axis=0)
        sum_ghat += out["Ghat"]
        M, P, Q = out["M"], out["Phat"], out["Q"]
        last = out
    E_T = last["E_next"]
    assert np.allclose(sum_g, sum_ghat + E_T.mean(axis=0), atol=1e-9)


def test_deferred_error_is_m_minus_ghat(psgd):
    rng = np.random.default_rng(8)
    W, r, shapes = 2, 3, [(20, 12)]
    dim = 240
    Q = rng.standard_normal(12 * r)
    a = psgd.lqsgd_step(rng.standard_normal((W, dim)), np.zeros((W, dim)), np.zeros(20 * r), Q,
                        shapes=shapes, rank=r, have_prev=False, seed=1, step=0)
    b = psgd.lqsgd_step(rng.standard_normal((W, dim)), a["M"], a["Phat"], a["Q"],
                        shapes=shapes, rank=r, have_prev=True, seed=1, step=1)
    assert np.allclose(b["E"], a["E_next"], atol=1e-12)


def test_log_quantizer_is_wired_in(psgd, oracle):
    rng = np.random.default_rng(9)
    W, r, shapes = 4, 4, [(64, 48), (32, 32)]
    G = _lowrank_workers(rng, W, shapes, r) + 1e-3 * rng.standard_normal(
        (W, sum(n * m for n, m in shapes)))
    Q0 = rng.standard_normal(sum(m * r for _, m in shapes))
    kw = dict(shapes=shapes, rank=r, have_prev=False, seed=5, step=3)
    ex = psgd.lqsgd_step(G, np.zeros_like(G), np.zeros(96 * r), Q0, lq=False, **kw)
    lq = psgd.lqsgd_step(G, np.zeros_like(G), np.zeros(96 * r), Q0, lq=True, **kw)
    rel = np.linalg.norm(lq["Ghat"] - ex["Ghat"]) / np.linalg.norm(ex["Ghat"])
    # near a factor's max, one log bin spans (1 + a) log(1 + a) / (127 a) ~ 2% of
    # the max, so each stochastically rounded factor is off by a few percent
    assert 0 < rel < 0.2
    psizes = np.array([n * r for n, _ in shapes])
    mx, codes = oracle.logq_quantize(lq["Pw"].astype(np.float32), psizes, seed=5, step=6)
    assert np.array_equal(codes, lq["lqP"]["codes"]) and np.array_equal(mx, lq["lqP"]["maxabs"])
    qsizes = np.array([m * r for _, m in shapes])
    mx, codes = oracle.logq_quantize(lq["Qw"].astype(np.float32), qsizes, seed=5, step=7)
    assert np.array_equal(codes, lq["lqQ"]["codes"])


def _round_f32(x):
    """Exact round-to-nearest-even of a Fraction to float32."""
    from fractions import Fraction
    f = np.float32(float(x))
    cands = [np.nextafter(f, np.float32(-np.inf)), f, np.nextafter(f, np.float32(np.inf))]
    best = min(cands, key=lambda c: (abs(Fraction(float(c)) - x),
                                     int(np.frombuffer(np.float32(c).tobytes(), np.uint32)[0]) & 1))
    return np.float32(best)


def test_lowrank_fma_is_a_chain_of_single_roundings(oracle):
    """Each entry of the float32 low-rank value is acc <- round(p_k q_k + acc)
    from acc = 0, every step one correct rounding of the exact value."""
    from fractions import Fraction
    rng = np.random.default_rng(11)
    P = (rng.standard_normal((6, 5)) * np.exp2(rng.integers(-20, 20, (6, 5)))).astype(np.float32)
    Q = (rng.standard_normal((7, 5)) * np.exp2(rng.integers(-20, 20, (7, 5)))).astype(np.float32)
    out = oracle.lowrank_fma(P, Q)
    for i in range(6):
        for j in range(7):
            acc = np.float32(0)
            for k in range(5):
                acc = _round_f32(Fraction(float(P[i, k])) * Fraction(float(Q[j, k]))
                                 + Fraction(float(acc)))
            assert acc == out[i, j], (i, j)
