"""Stage-by-stage checks of one PowerSGD + log-quantizer step against the
oracle, on the GPU's own input to each stage (shared by the single-GPU step
tests and the data-parallel exchange tests).  The tolerances and the reasons
for them are stated in tests/test_gpu_psgd.py."""
import numpy as np

U = 2.0 ** -24
ALPHA = 10.0


def host(t):
    return t.detach().cpu().numpy()


def mats(flat, rows, cols):
    out, off = [], 0
    for n, m in zip(rows, cols):
        out.append(flat[..., off:off + n * m].reshape(flat.shape[:-1] + (n, m)))
        off += n * m
    return out


def factors(flat, lens, r):
    out, off = [], 0
    for n in lens:
        out.append(flat[..., off:off + n * r].reshape(flat.shape[:-1] + (n, r)))
        off += n * r
    return out


def check_lq(oracle, x, sizes, seed, step, codes_gpu, max_gpu, sum_gpu):
    mx, codes = oracle.logq_quantize(x, sizes, alpha=ALPHA, seed=seed, step=step)
    assert np.array_equal(mx, max_gpu)
    diff = np.abs(codes.astype(np.int32) - codes_gpu.astype(np.int32))
    assert diff.max() <= 1
    assert (diff != 0).sum() <= max(1, int(1e-5 * diff.size))
    ref = oracle.logq_decode_sum(codes_gpu, max_gpu, sizes, alpha=ALPHA)
    off = 0
    for k, n in enumerate(sizes):
        tol = 1e-6 * float(max_gpu[:, k].sum())
        assert np.abs(sum_gpu[off:off + n] - ref[off:off + n]).max() <= tol
        off += n


def check_step(oracle, psgd, sh, W, g, s, have_prev, seed, step):
    """Every stage of one step against the oracle, on the GPU's own inputs."""
    r = sh.rank
    # state update, bit-exact
    for l, (n, m) in enumerate(zip(sh.rows, sh.cols)):
        gl = mats(g, sh.rows, sh.cols)[l]
        mi = mats(s["m_in"], sh.rows, sh.cols)[l]
        mo = mats(s["m"], sh.rows, sh.cols)[l]
        if have_prev:
            gh = oracle.lowrank_fma(factors(s["p_in"], sh.rows, r)[l],
                                    factors(s["q_in"], sh.cols, r)[l])
            e = (mi - gh[None]).astype(np.float32)
        else:
            e = mi
        assert np.array_equal((gl + e).astype(np.float32).view(np.uint32),
                              mo.view(np.uint32)), f"M of matrix {l}"
    # P_w = M Q within the bound of its fp32 sum order
    for l, (n, m) in enumerate(zip(sh.rows, sh.cols)):
        M = mats(s["m"], sh.rows, sh.cols)[l].astype(np.float64)
        Qm = factors(s["q_in"], sh.cols, r)[l].astype(np.float64)
        exact = M @ Qm
        bound = (-(-m // 32) + 6) * U * (np.abs(M) @ np.abs(Qm)) * 1.01 + 1e-30
        got = factors(s["pw"], sh.rows, r)[l]
        assert (np.abs(got - exact) <= bound).all(), f"P_w of matrix {l}"
    # log quantizer of the P_w and its decoded sum
    psizes = np.array([n * r for n in sh.rows], np.int64)
    check_lq(oracle, s["pw"], psizes, seed, 2 * step, s["codes_p"], s["max_p"], s["psum"])
    # orthonormalization
    for l, n in enumerate(sh.rows):
        ref = psgd.mgs(factors(s["psum"], sh.rows, r)[l])
        got = factors(s["phat"], sh.rows, r)[l].astype(np.float64)
        assert np.abs(got - ref).max() <= 1e-5, f"P_hat of matrix {l}"
        nz = np.linalg.norm(ref, axis=0) > 0
        gram = got[:, nz].T @ got[:, nz]
        assert np.abs(gram - np.eye(nz.sum())).max() <= 1e-5
    # Q_w = M^T P_hat within the bound of its fp32 sum order
    for l, (n, m) in enumerate(zip(sh.rows, sh.cols)):
        M = mats(s["m"], sh.rows, sh.cols)[l].astype(np.float64)
        Ph = factors(s["phat"], sh.rows, r)[l].astype(np.float64)
        exact = np.einsum("wnm,nr->wmr", M, Ph)
        bound = (n + 2) * U * np.einsum("wnm,nr->wmr", np.abs(M), np.abs(Ph)) * 1.01 + 1e-30
        got = factors(s["qw"], sh.cols, r)[l]
        assert (np.abs(got - exact) <= bound).all(), f"Q_w of matrix {l}"
    qsizes = np.array([m * r for m in sh.cols], np.int64)
    check_lq(oracle, s["qw"], qsizes, seed, 2 * step + 1, s["codes_q"], s["max_q"], s["qsum"])
    assert np.array_equal((s["qsum"] / np.float32(W)).astype(np.float32).view(np.uint32),
                          s["q"].view(np.uint32))
    # reconstruction, bit-exact
    for l in range(sh.nmats):
        gh = oracle.lowrank_fma(factors(s["phat"], sh.rows, r)[l], factors(s["q"], sh.cols, r)[l])
        assert np.array_equal(gh.view(np.uint32),
                              mats(s["ghat"], sh.rows, sh.cols)[l].view(np.uint32)), l
