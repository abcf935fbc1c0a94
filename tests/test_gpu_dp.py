"""The data-parallel exchange on the GPU through NCCL (one rank on this GPU).

With one rank holding all W workers, ``DataParallelStep`` runs the library's
kernels and two real NCCL all-reduces.  Every exchange is checked against the
oracle on the same rows: the scale within 1e-5 of the oracle's fp64 norm (the
max-abs scale exactly), and the mean and the error rows bit for bit given the
GPU's scale.  It must also equal the single-GPU fused step bit for bit (same
rows, same partition, so the same scale).  The LQ-SGD exchange is checked stage
by stage against oracle/psgd.py at the single-GPU step's tolerances.  Two or
more ranks need two or more GPUs; their host-side orchestration is covered by
tests/test_dp_exchange.py with gloo on CPU.
"""
import datetime

import numpy as np
import pytest
import torch
import torch.distributed as dist

import synthetic
from psgd_checks import check_step, host

pytestmark = pytest.mark.gpu


def _init_single_rank(tmp_path):
    """A one-rank NCCL group whose rendezvous is a file store: no TCP port
    that another process on the box could already hold."""
    store = dist.FileStore(str(tmp_path / "store"), 1)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))


@pytest.fixture(scope="module")
def gq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import allreduce_compatible_gradient_global_b200 as gq
    return gq


def check_against_oracle(oracle, cfg, g, e_before, step, scale, out, e_after):
    """One exchange step against the oracle's step on the same rows: the scale
    within 1e-5 of the fp64 norm (exact for max-abs), the mean and the error
    rows bit for bit given the GPU's scale.  g, e_before: host arrays."""
    W = g.shape[0]
    S = np.float32(scale)
    kw = dict(levels=0 if cfg.levels == "uniform" else 1, s=cfg.s, L=cfg.L,
              scale_kind=0 if cfg.scale_kind == "l2" else 1)
    ref = oracle.step(g, e_before, seed=cfg.seed, step=step, ef=cfg.ef, S=S, **kw)
    if kw["scale_kind"] == 0:
        assert abs(float(S) - float(ref["S"])) <= 1e-5 * float(ref["S"]), step
    else:
        assert S == ref["S"], step
    assert np.array_equal(out.view(np.uint32), ref["out"].view(np.uint32)), step
    if cfg.ef:
        assert np.array_equal(e_after.view(np.uint32), ref["e"].view(np.uint32)), step


@pytest.mark.parametrize("kw,ef", [(dict(s=15, bits=5, wire="int8"), False),
                                   (dict(levels="exp", L=5, bits=4, wire="int8",
                                         scale_kind="maxabs"), True),
                                   (dict(levels="exp", L=8, bits=5, wire="f16"), False),
                                   (dict(s=127, bits=8, wire="f16"), True)])
def test_nccl_single_rank_matches_oracle_and_fused_step(gq, oracle, kw, ef, tmp_path):
    from allreduce_compatible_gradient_global_b200.dp import DataParallelStep
    _init_single_rank(tmp_path)
    try:
        W, d = 4, 100_003
        cfg = gq.GQConfig(seed=7, ef=ef, **kw)
        g = synthetic.make_gradients(W, d, "student_t3", seed=1, device="cuda", seg=1000,
                                     lo=-4, hi=0)
        e1 = torch.zeros_like(g)
        e2 = torch.zeros_like(g)
        stepper = DataParallelStep(cfg, d, w_local=W)
        buf = gq.StepBuffers(cfg, W, d, ef=False)
        gh = host(g)
        for t in range(3):
            cfg.step = t
            e_before = host(e1) if ef else None
            out = stepper(g, e1, step=t, check=True).clone()
            check_against_oracle(oracle, cfg, gh, e_before, t, stepper.scale.item(), host(out),
                                 host(e1) if ef else None)
            gq.gq_step_fused(g, e2 if ef else None, cfg, buf.scale, buf.norms, buf.codes, buf.sum,
                             buf.out, buf.ws)
            assert gq.gq_get_device_status(buf.ws) == gq.GQ_OK
            torch.cuda.synchronize()
            assert torch.equal(stepper.scale, buf.scale)
            assert torch.equal(out.view(torch.int32), buf.out.view(torch.int32)), t
            if ef:
                assert torch.equal(e1, e2), t
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("r", [1, 5])
def test_nccl_single_rank_lqsgd_matches_oracle_and_whole_step(gq, oracle, r, tmp_path):
    """The LQ-SGD exchange (all-gather of the factor codes) on one NCCL rank
    holding all W workers: every stage against the oracle (oracle/psgd.py and
    the C log quantizer) on the exchange's own inputs to that stage, and the
    result equal to gq_lqsgd_step bit for bit, state included."""
    from oracle import psgd
    from allreduce_compatible_gradient_global_b200.dp import DataParallelLqsgdStep
    _init_single_rank(tmp_path)
    try:
        W = 4
        sh = gq.PsgdShapes([256, 100], [128, 64], r)

        def state():
            m = torch.zeros((W, sh.total), dtype=torch.float32, device="cuda")
            p = torch.zeros(sh.ptotal, dtype=torch.float32, device="cuda")
            q = synthetic.make_gradients(1, sh.qtotal, "normal", seed=3, device="cuda")[0]
            return m, p, q, torch.empty(sh.total, dtype=torch.float32, device="cuda")

        a, b = state(), state()
        ws = torch.empty(gq.gq_psgd_workspace_bytes(W, sh), dtype=torch.uint8, device="cuda")
        gq.gq_workspace_init(ws)
        dp = DataParallelLqsgdStep(sh, w_local=W, alpha=10.0, seed=12)
        psum = torch.empty(sh.ptotal, dtype=torch.float32, device="cuda")
        for t in range(3):
            g = synthetic.make_gradients(W, sh.total, "normal", seed=40 + t, device="cuda")
            snap = {"m_in": host(a[0]), "p_in": host(a[1]), "q_in": host(a[2])}
            dp(g, a[0], a[1], a[2], a[3], t > 0, t, check=True)
            # P before orthonormalization: the decode-sum of the gathered codes
            cfg = gq.GQConfig(levels="log", alpha=10.0, seed=12, step=2 * t)
            gq.gq_logq_decode_sum(dp.codes_p, dp.max_p, sh.rows, dp.ranks, cfg, psum)
            snap.update(m=host(a[0]), pw=host(dp.pw), codes_p=host(dp.codes_p),
                        max_p=host(dp.max_p), psum=host(psum), phat=host(a[1]), qw=host(dp.qw),
                        codes_q=host(dp.codes_q), max_q=host(dp.max_q), qsum=host(dp.qsum),
                        q=host(a[2]), ghat=host(a[3]))
            check_step(oracle, psgd, sh, W, host(g), snap, have_prev=t > 0, seed=12, step=t)
            gq.gq_lqsgd_step(g, b[0], sh, t > 0, gq.GQConfig(levels="log", alpha=10.0, seed=12,
                                                             step=t), b[1], b[2], b[3], ws)
            torch.cuda.synchronize()
            for x, y in zip(a, b):
                assert torch.equal(x, y), t
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("chunks,kw", [(4, dict(s=15, bits=5, wire="int8", ef=True)),
                                       (3, dict(levels="exp", L=8, bits=5, wire="f16"))])
def test_nccl_chunked_exchange_matches_oracle_and_unchunked(gq, oracle, chunks, kw, tmp_path):
    """Chunk k + 1 is quantized while chunk k is all-reduced (NCCL, async);
    with each chunk drawing the uniforms of its own coordinates the mean and
    the error buffer equal the oracle's step on the whole row and are
    bit-identical to the unchunked exchange."""
    from allreduce_compatible_gradient_global_b200.dp import DataParallelStep
    _init_single_rank(tmp_path)
    try:
        d = 1_000_003 - 3  # a multiple of 4, not of 128
        cfg = gq.GQConfig(seed=5, **kw)
        g = synthetic.make_gradients(1, d, "student_t3", seed=2, device="cuda", seg=4096,
                                     lo=-4, hi=0)
        e1, e2 = torch.zeros_like(g), torch.zeros_like(g)
        whole = DataParallelStep(cfg, d)
        parts = DataParallelStep(cfg, d, chunks=chunks)
        assert len(parts.bounds) == chunks
        gh = host(g)
        for t in range(2):
            e_before = host(e2) if cfg.ef else None
            a = whole(g, e1, step=t, check=True).clone()
            b = parts(g, e2, step=t, check=True).clone()
            torch.cuda.synchronize()
            check_against_oracle(oracle, cfg, gh, e_before, t, parts.scale.item(), host(b),
                                 host(e2) if cfg.ef else None)
            assert torch.equal(a.view(torch.int32), b.view(torch.int32)), t
            if cfg.ef:
                assert torch.equal(e1, e2), t
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("chunks,w_local,kw", [(1, 4, dict(s=15, bits=5, wire="int8", ef=True)),
                                               (3, 1, dict(s=15, bits=5, wire="int8", ef=True)),
                                               (4, 1, dict(levels="exp", L=8, bits=5,
                                                           wire="f16"))])
def test_nccl_graph_replay_matches_oracle_and_eager_exchange(gq, oracle, chunks, w_local, kw,
                                                           tmp_path):
    """The exchange captured once in a CUDA graph (kernels, NCCL all-reduces and,
    chunked, their overlap) and replayed with new gradients written in place
    equals the oracle's step and the eager exchange step for step, error
    buffers included; the graph advances the device step word itself."""
    from allreduce_compatible_gradient_global_b200.dp import DataParallelStep
    _init_single_rank(tmp_path)
    graphed = None
    try:
        d = 100_003
        cfg = gq.GQConfig(seed=5, **kw)
        eager = DataParallelStep(cfg, d, w_local=w_local, chunks=chunks)
        graphed = DataParallelStep(cfg, d, w_local=w_local, chunks=chunks)
        e1 = torch.zeros((w_local, d), dtype=torch.float32, device="cuda")
        e2 = torch.zeros_like(e1)
        g_in = torch.zeros_like(e1)
        graphed.capture(g_in, e2 if cfg.ef else None, first_step=2)
        assert torch.count_nonzero(e2) == 0  # the warm-up left the error rows alone
        for t in range(2, 6):
            g = synthetic.make_gradients(w_local, d, "student_t3", seed=100 + t, device="cuda",
                                         seg=1000, lo=-4, hi=0)
            g_in.copy_(g)
            e_before = host(e2) if cfg.ef else None
            got = graphed.replay(check=True).clone()
            want = eager(g, e1, step=t, check=True).clone()
            torch.cuda.synchronize()
            check_against_oracle(oracle, cfg, host(g), e_before, t, graphed.scale.item(),
                                 host(got), host(e2) if cfg.ef else None)
            assert torch.equal(got.view(torch.int32), want.view(torch.int32)), t
            if cfg.ef:
                assert torch.equal(e1, e2), t
        assert int(graphed.step_dev.item()) == 6
    finally:
        if graphed is not None:
            graphed.close()
        dist.destroy_process_group()


@pytest.mark.parametrize("W,sharded", [(4, False), (1, True)])
def test_nccl_single_rank_natural_exchange_matches_the_oracle(gq, oracle, W, sharded, tmp_path):
    """DataParallelNatStep on one NCCL rank (all W workers gathered, or one
    worker through the all-to-all of the sharded form): the codes and the
    decoded sum equal the oracle's, bit for bit."""
    from allreduce_compatible_gradient_global_b200.dp import DataParallelNatStep
    _init_single_rank(tmp_path)
    try:
        n = 50_001
        x = synthetic.make_gradients(W, n, "student_t3", seed=8, device="cuda", seg=100, lo=-25,
                                     hi=2)
        step = DataParallelNatStep(n, w_local=W, seed=21, sharded=sharded)
        for t in range(2):
            out = step(x, t, check=True).clone()
            ref = oracle.nat_quantize(x.cpu().numpy(), seed=21, step=t)
            assert np.array_equal(step.codes_l.cpu().numpy().view(np.uint16), ref)
            want = oracle.nat_decode_sum(ref)
            assert np.array_equal(out.cpu().numpy().view(np.uint32), want.view(np.uint32)), t
    finally:
        dist.destroy_process_group()

