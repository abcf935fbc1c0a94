"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Bars (the method's own): integer codes, packed bytes and integer sums
bit-exact; decoded means and error-feedback buffers bit-exact when the oracle
is given the GPU's scale; the scale within 1e-5 relative of the oracle's fp64
norm (exact for max-abs).  Small cases span several 128-coordinate blocks and
ragged tails; the full-size workloads are checked on sampled blocks in the
launch configuration the benchmark times.
"""
import math

import numpy as np
import pytest
import torch

import synthetic

pytestmark = pytest.mark.gpu

SCALE_RTOL = 1e-5


@pytest.fixture(scope="module")
def gq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import allreduce_compatible_gradient_global_b200 as gq
    return gq


def oracle_kw(cfg):
    return dict(levels=0 if cfg.levels == "uniform" else 1, s=cfg.s, L=cfg.L)


def gpu_step(gq, g, e, cfg, split=False):
    """Run the path on device tensors; returns host copies of every output."""
    W, d = g.shape
    buf = gq.StepBuffers(cfg, W, d, device=g.device, ef=False)
    e_dev = e.clone() if e is not None else None
    gq.gq_global_norm(g, e_dev if cfg.ef else None, cfg, buf.scale, buf.norms, buf.ws)
    if not split:
        gq.gq_quantize_aggregate(g, e_dev, cfg, buf.scale, buf.codes, buf.sum, buf.out, buf.ws)
    else:
        gq.gq_quantize_pack(g, e_dev, cfg, buf.scale, buf.codes, buf.ws)
        gq.gq_aggregate(buf.codes, W, d, cfg, buf.sum, buf.ws)
        gq.gq_dequantize_ef(buf.sum, buf.codes, g, e_dev, W, d, cfg, buf.scale, buf.out, buf.ws)
    assert gq.gq_get_device_status(buf.ws) == gq.GQ_OK
    torch.cuda.synchronize()
    return dict(S=np.float32(buf.scale.item()), norms=buf.norms.cpu().numpy(),
                codes=buf.codes.cpu().numpy(), sum=buf.sum.cpu().numpy().astype(np.int32),
                out=buf.out.cpu().numpy(),
                e=None if e_dev is None else e_dev.cpu().numpy())


def check_against_oracle(oracle, cfg, g, e, r):
    """Compare GPU results r with the oracle on host copies g, e."""
    kw = oracle_kw(cfg)
    sk = oracle.SCALE_L2 if cfg.scale_kind == "l2" else oracle.SCALE_MAXABS
    S_ref, norms_ref = oracle.global_scale(g, e if cfg.ef else None, sk)
    if sk == oracle.SCALE_L2:
        assert abs(float(r["S"]) - float(S_ref)) <= SCALE_RTOL * float(S_ref) + 1e-38
        assert np.allclose(r["norms"], norms_ref, rtol=SCALE_RTOL, atol=1e-30)
    else:
        assert r["S"] == S_ref
        assert np.array_equal(r["norms"], norms_ref)
    ref = oracle.step(g, e if cfg.ef else None, scale_kind=sk, seed=cfg.seed, step=cfg.step,
                      ef=cfg.ef, bits=cfg.bits, S=r["S"], **kw)
    assert np.array_equal(r["codes"], ref["packed"]), "packed codes differ"
    assert np.array_equal(r["sum"], ref["sum"]), "integer sums differ"
    assert np.array_equal(r["out"].view(np.uint32), ref["out"].view(np.uint32)), "means differ"
    if cfg.ef:
        assert np.array_equal(r["e"].view(np.uint32), ref["e"].view(np.uint32)), "EF differs"
    return ref


CASES = [
    # (W, d, cfg kwargs)
    (4, 1, dict(s=15, bits=5, wire="int8")),
    (4, 3, dict(s=15, bits=5, wire="int8")),
    (4, 33, dict(s=15, bits=5, wire="int8")),
    (4, 127, dict(s=15, bits=5, wire="int8")),
    (4, 128, dict(s=15, bits=5, wire="int8")),
    (4, 129, dict(s=15, bits=5, wire="int8")),
    (4, 4099, dict(s=15, bits=5, wire="int8")),            # d % 4 == 3: scalar rows
    (4, 65536 + 44, dict(s=15, bits=5, wire="int8")),      # ragged last block, vector rows
    (4, 1 << 18, dict(s=15, bits=5, wire="int8")),
    (8, 20000, dict(s=15, bits=5, wire="int8")),
    (8, 20002, dict(s=7, bits=4, wire="int8", seed=3)),
    (3, 10001, dict(s=7, bits=4, wire="int8", step=9)),    # W not a power of two
    (8, 30000, dict(s=127, bits=8, wire="int16", seed=11)),
    (5, 7777, dict(s=1000, bits=16, wire="int16")),
    (1, 5000, dict(s=3, bits=4, wire="int8")),
    (8, 40000, dict(levels="exp", L=8, bits=5, wire="int16", scale_kind="maxabs")),
    (8, 40001, dict(levels="exp", L=8, bits=5, wire="int16", scale_kind="l2", seed=5)),
    (2, 3333, dict(levels="exp", L=3, bits=4, wire="int8", step=2)),
    (4, 12345, dict(levels="exp", L=13, bits=5, wire="int16")),
    (1, 2222, dict(levels="exp", L=15, bits=5, wire="int16")),
    (4, 9000, dict(s=15, bits=5, wire="int8", scale_kind="maxabs")),
    (12, 5000, dict(s=2, bits=4, wire="int8", seed=0xFFFFFFFFFFFFFFFF, step=0xFFFFFFFF)),
    (40, 8192, dict(s=3, bits=4, wire="int8")),           # rows too many to stage: register path
    (16, 50000, dict(s=7, bits=4, wire="int8", seed=8)),  # 16 staged rows
    (8, 1 << 20, dict(s=15, bits=5, wire="int8", seed=9)),  # many tiles per block
    (8, 30001, dict(s=127, bits=8, wire="f16", seed=12)),   # fp16 sums, ragged tail
    (8, 40000, dict(levels="exp", L=8, bits=5, wire="f16", scale_kind="maxabs")),
    (16, 5003, dict(s=127, bits=8, wire="f16")),            # |sum| up to 2032
]


@pytest.mark.parametrize("W,d,kw", CASES)
def test_fused_step_matches_oracle(gq, oracle, W, d, kw):
    cfg = gq.GQConfig(**{"seed": 1234, **kw})
    g = synthetic.make_gradients(W, d, "student_t3", seed=W * 7919 + d, device="cuda",
                                 seg=1000, lo=-4, hi=0)
    r = gpu_step(gq, g, None, cfg)
    check_against_oracle(oracle, cfg, g.cpu().numpy(), None, r)


@pytest.mark.parametrize("W,d,kw", [c for c in CASES if c[1] in (33, 4099, 65580, 40000, 7777, 30001)])
def test_split_pipeline_equals_fused(gq, oracle, W, d, kw):
    cfg = gq.GQConfig(**{"seed": 99, **kw})
    g = synthetic.make_gradients(W, d, "laplace", seed=d, device="cuda", seg=512, lo=-5, hi=-2)
    fused = gpu_step(gq, g, None, cfg)
    split = gpu_step(gq, g, None, cfg, split=True)
    for k in ("codes", "sum", "out"):
        assert np.array_equal(fused[k], split[k]), k
    check_against_oracle(oracle, cfg, g.cpu().numpy(), None, split)


@pytest.mark.parametrize("split", [False, True])
@pytest.mark.parametrize("W,d,kw", [
    (8, 30000, dict(s=127, bits=8, wire="int16")),
    (4, 4097, dict(s=15, bits=5, wire="int8")),
    (8, 20000, dict(levels="exp", L=8, bits=5, wire="int16", scale_kind="maxabs")),
    (16, 5003, dict(s=127, bits=8, wire="f16")),
    (3, 10001, dict(levels="exp", L=5, bits=4, wire="int8", scale_kind="l2")),  # generic W
    (4, 12345, dict(levels="exp", L=13, bits=5, wire="int16", scale_kind="l2")),
])
def test_error_feedback_steps_match_oracle(gq, oracle, W, d, kw, split):
    cfg = gq.GQConfig(**{"ef": True, "seed": 77, **kw})
    e_gpu = torch.zeros((W, d), dtype=torch.float32, device="cuda")
    e_ref = np.zeros((W, d), np.float32)
    for t in range(3):
        cfg.step = t
        g = synthetic.make_gradients(W, d, "normal_seg", seed=100 + t, device="cuda", seg=999,
                                     lo=-4, hi=0)
        r = gpu_step(gq, g, e_gpu, cfg, split=split)
        ref = check_against_oracle(oracle, cfg, g.cpu().numpy(), e_ref, r)
        e_gpu = torch.from_numpy(r["e"]).cuda()
        e_ref = ref["e"]


@pytest.mark.parametrize("ef", [False, True])
@pytest.mark.parametrize("W,d,kw", [
    (8, 1 << 20, dict(s=127, bits=8, wire="int16")),       # whole tiles, unrolled W
    (8, 30001, dict(s=127, bits=8, wire="int16")),         # ragged tail
    (3, 10001, dict(s=7, bits=4, wire="int8")),            # generic W
    (8, 40001, dict(levels="exp", L=8, bits=5, wire="int16", scale_kind="maxabs")),
    (5, 7001, dict(levels="exp", L=6, bits=4, wire="int16", scale_kind="l2")),
])
def test_fused_pass_without_codes_matches_oracle(gq, oracle, W, d, kw, ef):
    """With no code buffer the fused pass writes only the sums, the means and
    the error-feedback buffer; those match the oracle bit for bit."""
    cfg = gq.GQConfig(**{"ef": ef, "seed": 4242, "step": 3, **kw})
    g = synthetic.make_gradients(W, d, "normal_seg", seed=d + W, device="cuda", seg=777,
                                 lo=-4, hi=0)
    e0 = (0.01 * synthetic.make_gradients(W, d, "normal", seed=d + 1, device="cuda")
          if ef else None)
    buf = gq.StepBuffers(cfg, W, d, codes=False, ef=False)
    e_dev = e0.clone() if ef else None
    gq.gq_global_norm(g, e_dev, cfg, buf.scale, buf.norms, buf.ws)
    gq.gq_quantize_aggregate(g, e_dev, cfg, buf.scale, None, buf.sum, buf.out, buf.ws)
    assert gq.gq_get_device_status(buf.ws) == gq.GQ_OK
    torch.cuda.synchronize()
    S = np.float32(buf.scale.item())
    sk = oracle.SCALE_L2 if cfg.scale_kind == "l2" else oracle.SCALE_MAXABS
    e_host = e0.cpu().numpy() if ef else None
    ref = oracle.step(g.cpu().numpy(), e_host, scale_kind=sk, seed=cfg.seed, step=cfg.step,
                      ef=ef, bits=cfg.bits, S=S, **oracle_kw(cfg))
    assert np.array_equal(buf.sum.cpu().numpy().astype(np.int32), ref["sum"]), "integer sums differ"
    assert np.array_equal(buf.out.cpu().numpy().view(np.uint32), ref["out"].view(np.uint32))
    if ef:
        assert np.array_equal(e_dev.cpu().numpy().view(np.uint32), ref["e"].view(np.uint32))


def test_zero_input_and_empty(gq, oracle):
    cfg = gq.GQConfig(s=15, bits=5, wire="int8")
    g = torch.zeros((4, 1000), device="cuda")
    r = gpu_step(gq, g, None, cfg)
    assert r["S"] == 0 and not r["sum"].any() and not r["out"].any()
    assert np.array_equal(r["codes"], oracle.pack(np.zeros((4, 1000), np.int32), 5))
    g0 = torch.zeros((4, 0), device="cuda")
    buf = gq.StepBuffers(cfg, 4, 0)
    gq.gq_global_norm(g0, None, cfg, buf.scale, buf.norms, buf.ws)
    torch.cuda.synchronize()
    assert buf.scale.item() == 0.0


def test_nonfinite_input_sets_the_device_flag(gq):
    for kind in ("l2", "maxabs"):
        cfg = gq.GQConfig(s=15, bits=5, wire="int8", scale_kind=kind)
        g = torch.randn((4, 5000), device="cuda")
        g[2, 1234] = float("nan")
        buf = gq.StepBuffers(cfg, 4, 5000)
        gq.gq_step_fused(g, None, cfg, buf.scale, buf.norms, buf.codes, buf.sum, buf.out, buf.ws)
        assert gq.gq_get_device_status(buf.ws) == gq.GQ_ERR_NONFINITE
        # the flag is cleared by the read; a clean step afterwards reports OK
        g[2, 1234] = 0.0
        gq.gq_step_fused(g, None, cfg, buf.scale, buf.norms, buf.codes, buf.sum, buf.out, buf.ws)
        assert gq.gq_get_device_status(buf.ws) == gq.GQ_OK
        g[1, 7] = float("inf")
        gq.gq_step_fused(g, None, cfg, buf.scale, buf.norms, buf.codes, buf.sum, buf.out, buf.ws)
        assert gq.gq_get_device_status(buf.ws) == gq.GQ_ERR_NONFINITE


def test_repeatable_bit_for_bit(gq):
    cfg = gq.GQConfig(s=15, bits=5, wire="int8", seed=5)
    g = synthetic.make_gradients(8, 300000, "student_t3", seed=1, device="cuda", seg=4096,
                                 lo=-4, hi=-1)
    a = gpu_step(gq, g, None, cfg)
    b = gpu_step(gq, g, None, cfg)
    for k in ("codes", "sum", "out", "norms"):
        assert np.array_equal(a[k], b[k]), k
    assert a["S"] == b["S"]


def test_host_buffer_step_equals_device_step(gq):
    cfg = gq.GQConfig(s=15, bits=5, wire="int8", seed=21)
    W, d = 4, 100000
    g = synthetic.make_gradients(W, d, "normal", seed=3, device="cuda")
    dev = gpu_step(gq, g, None, cfg)
    g_host = g.cpu().pin_memory()
    out_host = torch.empty(d, dtype=torch.float32).pin_memory()
    scale_host = torch.empty(1, dtype=torch.float32).pin_memory()
    buf = gq.StepBuffers(cfg, W, d)
    g_dev = torch.empty_like(g)
    gq.gq_step_fused_host(g_host, g_dev, None, cfg, buf.scale, buf.codes, buf.sum, buf.out,
                          out_host, scale_host, buf.ws)
    torch.cuda.current_stream().synchronize()
    assert np.array_equal(out_host.numpy(), dev["out"])
    assert scale_host.item() == dev["S"]


# ------------------------------------------------------------------ LQ-SGD
@pytest.mark.parametrize("rank", [1, 4, 7])
def test_logq_matches_oracle(gq, oracle, rank):
    W = synthetic.LQ_WORKLOAD["W"]
    alpha = synthetic.LQ_WORKLOAD["alpha"]
    x, sizes = synthetic.lq_factors(rank, W=W, device="cuda")
    rows = [4096] * len(sizes)
    cols = [rank] * len(sizes)
    cfg = gq.GQConfig(levels="log", alpha=alpha, seed=4242, step=3)
    n = x.shape[1]
    maxabs = torch.empty((W, len(sizes)), dtype=torch.float32, device="cuda")
    codes = torch.empty((W, n), dtype=torch.int8, device="cuda")
    out = torch.empty(n, dtype=torch.float32, device="cuda")
    ws = torch.empty(gq.gq_workspace_bytes(gq.GQConfig(), W, 1), dtype=torch.uint8, device="cuda")
    gq.gq_workspace_init(ws)
    gq.gq_logq_quantize(x, rows, cols, cfg, maxabs, codes, ws)
    gq.gq_logq_decode_sum(codes, maxabs, rows, cols, cfg, out)
    assert gq.gq_get_device_status(ws) == gq.GQ_OK
    xh = x.cpu().numpy()
    mx_ref, codes_ref = oracle.logq_quantize(xh, sizes, alpha=alpha, seed=4242, step=3)
    out_ref = oracle.logq_decode_sum(codes_ref, mx_ref, sizes, alpha=alpha)
    mx, c, o = maxabs.cpu().numpy(), codes.cpu().numpy().astype(np.int32), out.cpu().numpy()
    assert np.array_equal(mx, mx_ref)
    diff = np.abs(c - codes_ref.astype(np.int32))
    assert diff.max() <= 1
    assert (diff != 0).sum() <= max(1, math.floor(1e-5 * diff.size)), (diff != 0).sum()
    # decoded sums: entries whose W codes all agree are within W * 1e-6 * max|factor|
    agree = (diff == 0).all(axis=0)
    mcol = np.concatenate([np.repeat(mx_ref[:, m:m + 1], s, axis=1)
                           for m, s in enumerate(sizes)], axis=1)
    tol = 1e-6 * mcol.sum(axis=0)
    assert np.all(np.abs(o - out_ref)[agree] <= tol[agree])
    # where a code moved by one bin, the sum moves by at most one bin width
    assert np.all(np.abs(o - out_ref)[~agree] <= 0.03 * mcol.max(axis=0)[~agree] + tol[~agree])


def test_bounded_wait_reports_timeout_and_context_survives(gq):
    cfg = gq.GQConfig(s=15, bits=5, wire="int8", seed=3)
    buf = gq.StepBuffers(cfg, 8, 100000)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    assert gq.gq_selftest_wait_timeout(buf.ws, 50) == gq.GQ_ERR_TIMEOUT
    t1.record()
    torch.cuda.synchronize()
    assert 40.0 <= t0.elapsed_time(t1) < 5000.0
    # the flag was cleared by the read, and the device still runs the path
    g = synthetic.make_gradients(8, 100000, "normal", seed=1, device="cuda")
    gq.gq_step_fused(g, None, cfg, buf.scale, buf.norms, buf.codes, buf.sum, buf.out, buf.ws)
    assert gq.gq_get_device_status(buf.ws) == gq.GQ_OK


@pytest.mark.parametrize("d", [4000, 4001])
def test_rounding_decision_boundaries(gq, oracle, d):
    """Inputs placed a fraction of an ulp from the round-up boundary u = 1 - p
    (both sides, and on it), with S = s so the multiplier is exactly 1: the
    GPU's codes are floor(r + u) exactly, like the oracle's."""
    s, seed, step = 15, 7, 1
    cfg = gq.GQConfig(s=s, bits=5, wire="int8", seed=seed, step=step)
    v = np.zeros(d, np.float32)
    n = 0
    for j in range(d):
        f = oracle.uniform_bits(seed, 0, step, 0, j)
        if (1 << 20) <= f < (1 << 21):
            u = f / float(1 << 23)
            v[j] = -(u + 2.0 ** -26) if n % 3 == 0 else (-(u - 2.0 ** -26) if n % 3 == 1 else -u)
            n += 1
    assert n > 300
    g = torch.from_numpy(v[None, :]).cuda()
    scale = torch.tensor([float(s)], dtype=torch.float32, device="cuda")
    codes = torch.empty((1, gq.gq_packed_row_bytes(cfg, d)), dtype=torch.uint8, device="cuda")
    ws = torch.empty(gq.gq_workspace_bytes(cfg, 1, d), dtype=torch.uint8, device="cuda")
    gq.gq_workspace_init(ws)
    gq.gq_quantize_pack(g, None, cfg, scale, codes, ws)
    assert gq.gq_get_device_status(ws) == gq.GQ_OK
    ref = oracle.quantize(v[None, :], s=s, seed=seed, step=step, S=np.float32(s))
    assert (ref == -1).sum() >= 100
    assert np.array_equal(codes.cpu().numpy(), oracle.pack(ref, 5))


@pytest.mark.parametrize("W,d,c0,n", [(4, 10000, 4096, 3000), (8, 65536, 1024, 40000),
                                      (3, 20001, 4, 999)])
def test_coordinate_offset_equals_the_whole_vector(gq, W, d, c0, n):
    """A chunk quantized with coord0 = its first coordinate (and the whole
    vector's scale) gives the same integer sums and means as those columns of
    the whole vector."""
    cfg = gq.GQConfig(s=15, bits=5, wire="int8", seed=31, step=2)
    g = synthetic.make_gradients(W, d, "normal", seed=d, device="cuda")
    whole = gq.StepBuffers(cfg, W, d)
    gq.gq_step_fused(g, None, cfg, whole.scale, whole.norms, whole.codes, whole.sum, whole.out,
                     whole.ws)
    chunk = g[:, c0:c0 + n].contiguous()
    part = gq.StepBuffers(cfg, W, n)
    cfgc = gq.GQConfig(s=15, bits=5, wire="int8", seed=31, step=2, coord0=c0)
    gq.gq_quantize_aggregate(chunk, None, cfgc, whole.scale, part.codes, part.sum, part.out,
                             part.ws)
    assert gq.gq_get_device_status(part.ws) == gq.GQ_OK
    torch.cuda.synchronize()
    assert torch.equal(part.sum, whole.sum[c0:c0 + n])
    assert torch.equal(part.out.view(torch.int32), whole.out[c0:c0 + n].view(torch.int32))
