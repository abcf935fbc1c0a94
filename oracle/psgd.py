"""PowerSGD low-rank step with LQ-SGD's log quantizer on both factors.

TEST INFRASTRUCTURE ONLY: imported by the tests, ``__graft_entry__.smoke()``
and the benchmark's CPU-baseline leg, never by the product package.

What it follows:

* "Trustworthy Efficient Communication for Distributed Learning using LQ-SGD
  Algorithm" (review, "What carries the argument"): the gradient matrix is
  approximated as G ~ P Q^T with PowerSGD's low-rank step, P and Q are each
  log-quantized before their All-Reduce, and the error E_t = G'_t - Ghat_t is
  added back on the next step; (Desk Editor's Note, "What is actually new"):
  both factors are log-quantized, with orthonormalization and error feedback;
  (referee comment on Section III-A): Ghat_t is the approximate global
  gradient used in place of g_t.
* PowerSGD (Vogels, Karimireddy and Jaggi, NeurIPS 2019, cited on that page),
  the published method: per matrix, with the previous step's Q as warm start,
  P_w = M_w Q, P = all-reduce(P_w), P_hat = orthonormalize(P),
  Q_w = M_w^T P_hat, Q = mean(Q_w), Ghat = P_hat Q^T, E_w = M_w - Ghat.

Readings taken where the pages are silent (each also stated where the GPU path
implements it):

* The all-reduce of P is a sum (orthonormalization does not depend on the
  column scale); the all-reduce of Q is a mean, so Ghat estimates the mean
  gradient.
* Orthonormalization is modified Gram-Schmidt over the columns in order; a
  column whose remaining norm is 0 stays 0.
* Each worker's P_w is log-quantized before the All-Reduce of P, and each
  worker's Q_w, computed from the orthonormalized P, before the All-Reduce of
  Q ("applied independently to P and Q before All-Reduce").
* The log quantizer is the one of ``oracle.logq_quantize`` (per worker and
  matrix max-abs, 8-bit codes); P draws its uniforms with step 2t and Q with
  step 2t + 1, so the two factors of one step never share a random stream.

Arithmetic is float64 (numpy matmul as the library primitive), except that the
factors pass through the float32 log quantizer, as on the wire.
"""
import numpy as np

from . import logq_decode_sum, logq_quantize


def split(flat, shapes):
    """Views of the matrices stored back to back (row-major) in flat[W][n]."""
    out, off = [], 0
    for (n, m) in shapes:
        out.append(flat[..., off:off + n * m].reshape(flat.shape[:-1] + (n, m)))
        off += n * m
    return out


def join(mats, W):
    """Inverse of split for a list of [W][n][m] arrays."""
    return np.concatenate([x.reshape(W, -1) for x in mats], axis=1)


def mgs(P):
    """Modified Gram-Schmidt on the columns of P (n x r), in column order:
    normalize column k, then remove its component from every later column.  A
    column whose remaining norm is 0 is left 0.  Returns a new array."""
    P = np.array(P, dtype=np.float64)
    r = P.shape[1]
    for k in range(r):
        nrm = np.sqrt(np.dot(P[:, k], P[:, k]))
        if nrm > 0:
            P[:, k] /= nrm
        for k2 in range(k + 1, r):
            P[:, k2] -= np.dot(P[:, k], P[:, k2]) * P[:, k]
    return P


def lq_factor_sum(X, sizes, *, alpha, seed, step):
    """Each worker's factors log-quantized and decoded, summed over workers:
    the on-GPU stand-in for the All-Reduce of one factor.  X: [W][sum(sizes)]."""
    mx, codes = logq_quantize(np.asarray(X, np.float32), sizes, alpha=alpha, seed=seed,
                              step=step)
    return dict(maxabs=mx, codes=codes,
                sum=logq_decode_sum(codes, mx, sizes, alpha=alpha).astype(np.float64))


def lqsgd_step(G, M_state, P_state, Q_state, *, shapes, rank, have_prev, alpha=10.0, seed=0,
               step=0, lq=True):
    """One step for W workers over a list of matrices.

    G, M_state: [W][sum n_l m_l] (M_state is the previous step's M when
    have_prev, else the initial error E, usually 0); P_state: [sum n_l r] (the
    previous P_hat, used only when have_prev); Q_state: [sum m_l r] (warm start,
    the previous mean Q).  lq=False replaces the log quantizer by the identity
    (exact sums), for the pins.

    Returns every intermediate: E (the error added back), M, Pw, P (sum), Phat,
    Qw, Q (mean), Ghat [sum n_l m_l], E_next (M - Ghat per worker), and the LQ
    codes and max-abs of both factors."""
    G = np.asarray(G, np.float64)
    W = G.shape[0]
    r = rank
    Ms = split(np.asarray(M_state, np.float64), shapes)
    Gs = split(G, shapes)
    Pst = split(np.asarray(P_state, np.float64)[None], [(n, r) for n, _ in shapes])
    Qst = split(np.asarray(Q_state, np.float64)[None], [(m, r) for _, m in shapes])
    E_l, M_l, Pw_l = [], [], []
    for l in range(len(shapes)):
        E = Ms[l] - (Pst[l][0] @ Qst[l][0].T)[None] if have_prev else Ms[l]
        M = Gs[l] + E
        E_l.append(E)
        M_l.append(M)
        Pw_l.append(M @ Qst[l][0])                     # [W][n][r]
    Pw = join(Pw_l, W)
    psizes = np.array([n * r for n, _ in shapes], np.int64)
    qsizes = np.array([m * r for _, m in shapes], np.int64)
    lqP = lq_factor_sum(Pw, psizes, alpha=alpha, seed=seed, step=2 * step) if lq else None
    P = lqP["sum"] if lq else Pw.sum(axis=0)
    P_l = split(P[None], [(n, r) for n, _ in shapes])
    Phat_l = [mgs(p[0]) for p in P_l]
    Qw_l = [np.einsum("wnm,nr->wmr", M_l[l], Phat_l[l]) for l in range(len(shapes))]
    Qw = join(Qw_l, W)
    lqQ = lq_factor_sum(Qw, qsizes, alpha=alpha, seed=seed, step=2 * step + 1) if lq else None
    Q = (lqQ["sum"] if lq else Qw.sum(axis=0)) / W
    Q_l = split(Q[None], [(m, r) for _, m in shapes])
    Ghat_l = [Phat_l[l] @ Q_l[l][0].T for l in range(len(shapes))]
    Ghat = join([g[None] for g in Ghat_l], 1)[0]
    E_next = join([M_l[l] - Ghat_l[l][None] for l in range(len(shapes))], W)
    return dict(E=join(E_l, W), M=join(M_l, W), Pw=Pw, P=P,
                Phat=join([p[None] for p in Phat_l], 1)[0], Qw=Qw, Q=Q, Ghat=Ghat,
                E_next=E_next, lqP=lqP, lqQ=lqQ)
