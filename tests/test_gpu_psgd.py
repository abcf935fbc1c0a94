"""GPU parity of the PowerSGD + log-quantizer step against the oracle.

Each stage is checked on the GPU's own input to that stage, so that a float
difference upstream cannot flip an integer decision downstream:

* element-wise results bit-exact: the state M = fl(G + fl(M_prev - Ghat)),
  the reconstruction Ghat (fma chain of the oracle's C helper) and the mean
  Q = fl(Q_sum / W);
* the log quantizer of both factors (the oracle's quantizer run on the GPU's
  P_w and Q_w) to the log quantizer's own bar, since the GPU's log1pf/expm1f
  and the host's may differ in the last place: max-abs exact, codes off by at
  most one bin on at most 1e-5 of the entries, decoded sums within
  1e-6 * sum_w max_w where the codes agree;
* reductions within the bound of their summation order: an fp32 sum of k
  terms, computed in any fixed order, is within k u sum |terms| of the exact
  sum (u = 2^-24); P_w sums m/32 lane terms then 5 butterfly levels, Q_w at
  most n rows (chunks included) -- both bounds are taken from the exact
  |terms| in fp64;
* orthonormalization within 1e-5 of the oracle's fp64 Gram-Schmidt of the
  same input, with the columns orthonormal to 1e-5;
* the whole-step call bit-identical to the split calls.
"""
import numpy as np
import pytest
import torch

import synthetic
from psgd_checks import ALPHA, U, check_step, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import allreduce_compatible_gradient_global_b200 as gq
    return gq


@pytest.fixture(scope="module")
def psgd(oracle):
    from oracle import psgd
    return psgd


class Run:
    """Device buffers of one configuration, and the split calls of one step."""

    def __init__(self, gq, W, rows, cols, r, seed):
        self.gq, self.W = gq, W
        self.sh = gq.PsgdShapes(rows, cols, r)
        sh = self.sh
        dev = "cuda"
        self.m = torch.zeros((W, sh.total), dtype=torch.float32, device=dev)
        self.p = torch.zeros(sh.ptotal, dtype=torch.float32, device=dev)
        self.q = synthetic.make_gradients(1, sh.qtotal, "normal", seed=seed + 1, device=dev)[0]
        self.pw = torch.empty((W, sh.ptotal), dtype=torch.float32, device=dev)
        self.qw = torch.empty((W, sh.qtotal), dtype=torch.float32, device=dev)
        self.qsum = torch.empty(sh.qtotal, dtype=torch.float32, device=dev)
        self.ghat = torch.empty(sh.total, dtype=torch.float32, device=dev)
        self.codes_p = torch.empty((W, sh.ptotal), dtype=torch.int8, device=dev)
        self.codes_q = torch.empty((W, sh.qtotal), dtype=torch.int8, device=dev)
        self.max_p = torch.empty((W, sh.nmats), dtype=torch.float32, device=dev)
        self.max_q = torch.empty((W, sh.nmats), dtype=torch.float32, device=dev)
        self.ws = torch.empty(gq.gq_psgd_workspace_bytes(W, sh), dtype=torch.uint8, device=dev)
        gq.gq_workspace_init(self.ws)
        self.rp = [r] * sh.nmats

    def split_step(self, g, have_prev, seed, step):
        gq, sh, W = self.gq, self.sh, self.W
        cfg = gq.GQConfig(levels="log", alpha=ALPHA, seed=seed, step=2 * step)
        snap = {"m_in": host(self.m), "p_in": host(self.p), "q_in": host(self.q)}
        gq.gq_psgd_project(g, self.m, sh, have_prev, self.p, self.q, self.pw)
        snap["m"], snap["pw"] = host(self.m), host(self.pw)
        gq.gq_logq_quantize(self.pw, sh.rows, self.rp, cfg, self.max_p, self.codes_p, self.ws)
        gq.gq_logq_decode_sum(self.codes_p, self.max_p, sh.rows, self.rp, cfg, self.p)
        snap["codes_p"], snap["max_p"], snap["psum"] = (host(self.codes_p), host(self.max_p),
                                                       host(self.p))
        gq.gq_psgd_orthonormalize(self.p, sh)
        snap["phat"] = host(self.p)
        gq.gq_psgd_back_project(self.m, self.p, sh, self.qw, self.ws)
        snap["qw"] = host(self.qw)
        cfg.step = 2 * step + 1
        gq.gq_logq_quantize(self.qw, sh.cols, self.rp, cfg, self.max_q, self.codes_q, self.ws)
        gq.gq_logq_decode_sum(self.codes_q, self.max_q, sh.cols, self.rp, cfg, self.qsum)
        snap["codes_q"], snap["max_q"], snap["qsum"] = (host(self.codes_q), host(self.max_q),
                                                       host(self.qsum))
        gq.gq_psgd_mean(self.qsum, self.q, W)
        snap["q"] = host(self.q)
        gq.gq_psgd_reconstruct(self.p, self.q, sh, self.ghat)
        snap["ghat"] = host(self.ghat)
        assert gq.gq_get_device_status(self.ws) == gq.GQ_OK
        return snap


SHAPES = [
    # (W, rows, cols, rank)
    (2, [64], [48], 1),
    (4, [100, 37, 1], [64, 20, 8], 4),          # ragged row tiles, a single-row matrix
    (3, [50, 33], [30, 7], 3),                  # some m % 4 != 0: scalar kernels
    (8, [256, 128], [512, 1024], 8),
    (2, [16] * 70, [32] * 70, 2),               # more matrices than one launch holds
    (4, [1500], [1028], 7),                     # several row chunks, a ragged column tile
]


@pytest.mark.parametrize("W,rows,cols,r", SHAPES)
def test_three_steps_match_oracle(gq, oracle, psgd, W, rows, cols, r):
    run = Run(gq, W, rows, cols, r, seed=W * 100 + r)
    for t in range(3):
        g = synthetic.make_gradients(W, run.sh.total, "normal", seed=1000 * t + r, device="cuda")
        s = run.split_step(g, have_prev=t > 0, seed=77, step=t)
        check_step(oracle, psgd, run.sh, W, host(g), s, have_prev=t > 0, seed=77, step=t)


@pytest.mark.parametrize("W,rows,cols,r", [SHAPES[1], SHAPES[3], SHAPES[2]])
def test_whole_step_equals_split_calls(gq, W, rows, cols, r):
    a = Run(gq, W, rows, cols, r, seed=5)
    b = Run(gq, W, rows, cols, r, seed=5)
    for t in range(2):
        g = synthetic.make_gradients(W, a.sh.total, "laplace", seed=t, device="cuda", seg=64,
                                     lo=-3, hi=0)
        a.split_step(g, have_prev=t > 0, seed=9, step=t)
        cfg = gq.GQConfig(levels="log", alpha=ALPHA, seed=9, step=t)
        gq.gq_lqsgd_step(g, b.m, b.sh, t > 0, cfg, b.p, b.q, b.ghat, b.ws)
        assert gq.gq_get_device_status(b.ws) == gq.GQ_OK
        for name in ("m", "p", "q", "ghat"):
            assert torch.equal(getattr(a, name), getattr(b, name)), (t, name)


def test_error_feedback_telescopes_on_gpu(gq):
    """sum_t mean_w G_t = sum_t Ghat_t + mean_w (M_T - Ghat_T), up to fp32 rounding."""
    W, rows, cols, r, T = 4, [96, 64], [128, 64], 2, 5
    run = Run(gq, W, rows, cols, r, seed=3)
    sg = torch.zeros(run.sh.total, dtype=torch.float64, device="cuda")
    sgh = torch.zeros_like(sg)
    for t in range(T):
        g = synthetic.make_gradients(W, run.sh.total, "normal", seed=50 + t, device="cuda")
        cfg = gq.GQConfig(levels="log", alpha=ALPHA, seed=4, step=t)
        gq.gq_lqsgd_step(g, run.m, run.sh, t > 0, cfg, run.p, run.q, run.ghat, run.ws)
        sg += g.double().mean(dim=0)
        sgh += run.ghat.double()
    e_T = run.m.double() - run.ghat.double()[None]
    resid = (sg - sgh - e_T.mean(dim=0)).abs().max().item()
    assert resid <= 1e-4 * max(1.0, sg.abs().max().item())


def test_host_side_errors(gq):
    bad = gq.PsgdShapes([4], [4], 9)
    with pytest.raises(gq.GQError):
        gq.gq_psgd_workspace_bytes(2, bad)
    sh = gq.PsgdShapes([8], [8], 2)
    g = torch.zeros((2, 64), dtype=torch.float32, device="cuda")
    m = torch.zeros_like(g)
    q = torch.zeros(16, dtype=torch.float32, device="cuda")
    pw = torch.zeros((2, 16), dtype=torch.float32, device="cuda")
    with pytest.raises(gq.GQError) as ei:  # have_prev without a previous P
        gq.gq_psgd_project(g, m, sh, True, None, q, pw)
    assert ei.value.status == gq.GQ_ERR_ARG
    ws = torch.zeros(gq.gq_psgd_workspace_bytes(2, sh), dtype=torch.uint8, device="cuda")
    p = torch.zeros(16, dtype=torch.float32, device="cuda")
    ghat = torch.zeros(64, dtype=torch.float32, device="cuda")
    with pytest.raises(gq.GQError) as ei:  # the step needs the log level set
        gq.gq_lqsgd_step(g, m, sh, False, gq.GQConfig(), p, q, ghat, ws)
    assert ei.value.status == gq.GQ_ERR_ARG


@pytest.mark.parametrize("r", [1, 7])
def test_full_size_lq_workload_sampled(gq, oracle, psgd, r):
    """The LQ-SGD workload (W = 8, 24 matrices of 4096 x 4096 per worker) for
    two steps through gq_lqsgd_step, with the split calls' stages checked on
    sampled rows and columns: M rows bit-exact, P_w rows and Q_w columns
    within their sum-order bounds, and P_hat orthonormal."""
    wl = synthetic.LQ_WORKLOAD
    W, L, n, m = wl["W"], wl["pairs"], wl["n"], wl["m"]
    sh = gq.PsgdShapes([n] * L, [m] * L, r)
    dev = "cuda"
    g = torch.empty((W, sh.total), dtype=torch.float32, device=dev)
    mst = torch.zeros_like(g)
    p = torch.zeros(sh.ptotal, dtype=torch.float32, device=dev)
    q = synthetic.make_gradients(1, sh.qtotal, "normal", seed=17, device=dev)[0]
    pw = torch.empty((W, sh.ptotal), dtype=torch.float32, device=dev)
    qw = torch.empty((W, sh.qtotal), dtype=torch.float32, device=dev)
    ghat = torch.empty(sh.total, dtype=torch.float32, device=dev)
    ws = torch.empty(gq.gq_psgd_workspace_bytes(W, sh), dtype=torch.uint8, device=dev)
    gq.gq_workspace_init(ws)
    rng = np.random.default_rng(r)
    for t in range(2):
        synthetic.fill_gradients(g, "normal", seed=900 + t)
        m_prev = {}
        picks = [(int(rng.integers(W)), int(rng.integers(L)), int(rng.integers(n)))
                 for _ in range(6)]
        for (w, l, i) in picks:
            off = l * n * m + i * m
            m_prev[(w, l, i)] = host(mst[w, off:off + m])
        p_prev, q_prev = host(p), host(q)
        # pass 1 alone, for its outputs; then the whole step from the same state
        m_copy = mst.clone()
        gq.gq_psgd_project(g, m_copy, sh, t > 0, p, q, pw)
        cfg = gq.GQConfig(levels="log", alpha=ALPHA, seed=21, step=t)
        gq.gq_lqsgd_step(g, mst, sh, t > 0, cfg, p, q, ghat, ws)
        assert gq.gq_get_device_status(ws) == gq.GQ_OK
        assert torch.equal(m_copy, mst)
        del m_copy
        for (w, l, i) in picks:
            off = l * n * m + i * m
            gr, mr = host(g[w, off:off + m]), host(mst[w, off:off + m])
            pl = p_prev[l * n * r:(l + 1) * n * r].reshape(n, r)
            ql = q_prev[l * m * r:(l + 1) * m * r].reshape(m, r)
            e = m_prev[(w, l, i)]
            if t > 0:
                e = (e - oracle.lowrank_fma(pl[i:i + 1], ql)[0]).astype(np.float32)
            assert np.array_equal((gr + e).astype(np.float32).view(np.uint32),
                                  mr.view(np.uint32)), (t, w, l, i)
            got = host(pw[w, l * n * r + i * r:l * n * r + (i + 1) * r])
            exact = mr.astype(np.float64) @ ql.astype(np.float64)
            bound = (m // 32 + 6) * U * (np.abs(mr).astype(np.float64) @
                                         np.abs(ql).astype(np.float64)) * 1.01
            assert (np.abs(got - exact) <= bound).all(), (t, w, l, i)
        ph = host(p).reshape(L, n, r).astype(np.float64)
        for l in range(L):
            assert np.abs(ph[l].T @ ph[l] - np.eye(r)).max() <= 1e-5
        # Q_w on sampled columns from the back projection of the final state
        gq.gq_psgd_back_project(mst, p, sh, qw, ws)
        for (w, l, _) in picks[:3]:
            j = int(rng.integers(m))
            col = host(mst[w, l * n * m + j:(l + 1) * n * m:m]).astype(np.float64)
            exact = col @ ph[l]
            bound = (n + 2) * U * (np.abs(col) @ np.abs(ph[l])) * 1.01
            got = host(qw[w, l * m * r + j * r:l * m * r + (j + 1) * r])
            assert (np.abs(got - exact) <= bound).all(), (t, w, l, j)
    del g, mst, ghat, ws
    torch.cuda.empty_cache()
