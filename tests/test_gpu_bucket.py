"""GPU parity of the per-bucket path against the oracle's bucket composition.

Bars, as for the global path: S_k within 1e-5 relative of the oracle's fp64
slice norm (exact for max-abs); the table's multiplier and unit are exactly
s/S_k rounded toward zero (or 1/S_k) and fl(S_k/s) (or S_k * 2^-(L-1)); packed
codes, integer sums, decoded means and error-feedback buffers bit-exact when
the oracle is given the GPU's S_k.  Cases span several buckets, ragged last
buckets, both fused kernels (d % 4 == 0 takes the bulk-copy pipeline, other d
the register path), both scale kernels (one launch up to 2^12-coordinate
buckets, chunk partials above), and buckets from 128 coordinates to more
than d.
"""
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
    return dict(levels=0 if cfg.levels == "uniform" else 1, s=cfg.s, L=cfg.L,
                scale_kind=0 if cfg.scale_kind == "l2" else 1)


def gpu_bucketed(gq, g, e, b, cfg, split=False):
    W, d = g.shape
    K = gq.gq_bucket_count(d, b)
    table = torch.full((3 * K,), -1.0, dtype=torch.float32, device=g.device)
    codes = torch.empty((W, gq.gq_packed_row_bytes(cfg, d)), dtype=torch.uint8, device=g.device)
    sum_ = torch.empty(d, dtype=cfg.wire_dtype, device=g.device)
    out = torch.empty(d, dtype=torch.float32, device=g.device)
    ws = torch.empty(gq.gq_bucket_workspace_bytes(cfg, W, d, b), dtype=torch.uint8,
                     device=g.device)
    gq.gq_workspace_init(ws)
    e_dev = e.clone() if e is not None else None
    if split:
        gq.gq_bucket_scales(g, e_dev if cfg.ef else None, b, cfg, table, ws)
        gq.gq_quantize_aggregate_bucketed(g, e_dev, b, cfg, table, codes, sum_, out, ws)
    else:
        gq.gq_step_bucketed(g, e_dev, b, cfg, table, codes, sum_, out, ws)
    status = gq.gq_get_device_status(ws)
    torch.cuda.synchronize()
    t = table.cpu().numpy()
    return dict(status=status, S=t[:K], mult=t[K:2 * K], unit=t[2 * K:],
                codes=codes.cpu().numpy(), sum=sum_.cpu().numpy().astype(np.int32),
                out=out.cpu().numpy(), e=None if e_dev is None else e_dev.cpu().numpy())


def check(oracle, cfg, g, e, b, r):
    kw = oracle_kw(cfg)
    ref_S = oracle.step_bucketed(g, e, bucket=1 << b, ef=cfg.ef, bits=None, **kw)["S"]
    if kw["scale_kind"] == 0:
        assert np.all(np.abs(r["S"].astype(np.float64) - ref_S) <= SCALE_RTOL * ref_S + 1e-38)
    else:
        assert np.array_equal(r["S"], ref_S)
    for k, Sk in enumerate(r["S"]):
        if cfg.levels == "uniform":
            want_a = oracle.uniform_multiplier(cfg.s, Sk) if Sk > 0 else np.float32(0)
            want_c = np.float32(Sk) / np.float32(cfg.s)
        else:
            want_a = oracle.uniform_multiplier(1, Sk) if Sk > 0 else np.float32(0)
            want_c = np.float32(Sk) * np.float32(2.0 ** -(cfg.L - 1))
        assert r["mult"][k] == want_a, k
        assert r["unit"][k] == want_c, k
    ref = oracle.step_bucketed(g, e, bucket=1 << b, seed=cfg.seed, step=cfg.step, ef=cfg.ef,
                               bits=cfg.bits, S=r["S"], **kw)
    assert np.array_equal(r["codes"], ref["packed"]), "packed codes differ"
    assert np.array_equal(r["sum"], ref["sum"]), "integer sums differ"
    assert np.array_equal(r["out"].view(np.uint32), ref["out"].view(np.uint32)), "means differ"
    if cfg.ef:
        assert np.array_equal(r["e"].view(np.uint32), ref["e"].view(np.uint32)), "EF differs"


CASES = [
    # (W, d, bucket_log2, cfg kwargs)
    (4, 10000, 10, dict(s=15, bits=5, wire="int8", ef=True)),
    (4, 10001, 10, dict(s=15, bits=5, wire="int8")),               # register path
    (8, 5 * 4096 + 256, 12, dict(s=15, bits=5, wire="int8")),
    (8, 3 * 8192 + 1000, 13, dict(s=127, bits=8, wire="int16", ef=True)),
    (3, 777, 7, dict(s=7, bits=4, wire="int8", step=4)),           # 128-coordinate buckets
    (8, 40000, 9, dict(levels="exp", L=8, bits=5, wire="int16", scale_kind="maxabs")),
    (8, 40002, 8, dict(levels="exp", L=8, bits=5, wire="int16", ef=True)),
    (5, 9000, 11, dict(s=1000, bits=16, wire="int16", scale_kind="maxabs")),
    (4, 3000, 14, dict(s=15, bits=5, wire="int8")),                # one bucket covers d
    (16, 50000, 10, dict(s=7, bits=4, wire="int8", seed=8)),
    (40, 8192, 10, dict(s=3, bits=4, wire="int8")),                # rows too many to stage
    (8, (1 << 20) + 4, 17, dict(s=15, bits=5, wire="int8", seed=9, ef=True)),
    (4, 40003, 14, dict(s=15, bits=5, wire="int8", ef=True, scale_kind="maxabs")),
    (3, 70001, 13, dict(levels="exp", L=6, bits=4, wire="int8", step=5)),
]


@pytest.mark.parametrize("W,d,b,kw", CASES)
def test_bucketed_step_matches_oracle(gq, oracle, W, d, b, kw):
    cfg = gq.GQConfig(**{"seed": 4321, **kw})
    g = synthetic.make_gradients(W, d, "student_t3", seed=W * 31 + d, device="cuda", seg=300,
                                 lo=-5, hi=0)
    e = (synthetic.make_gradients(W, d, "normal", seed=d + 7, device="cuda") * 1e-3
         if cfg.ef else None)
    r = gpu_bucketed(gq, g, e, b, cfg)
    assert r["status"] == gq.GQ_OK
    check(oracle, cfg, g.cpu().numpy(), None if e is None else e.cpu().numpy(), b, r)


def test_split_calls_equal_step(gq):
    W, d, b = 8, 30000, 11
    cfg = gq.GQConfig(s=15, bits=5, wire="int8", ef=True, seed=3)
    g = synthetic.make_gradients(W, d, "laplace", seed=1, device="cuda", seg=100, lo=-4, hi=0)
    e = synthetic.make_gradients(W, d, "normal", seed=2, device="cuda") * 1e-4
    a = gpu_bucketed(gq, g, e, b, cfg)
    c = gpu_bucketed(gq, g, e, b, cfg, split=True)
    for key in ("S", "mult", "unit", "codes", "sum", "out", "e"):
        assert np.array_equal(a[key], c[key]), key


def test_zero_and_huge_buckets(gq, oracle):
    W, d, b = 4, 4096, 10
    cfg = gq.GQConfig(s=15, bits=5, wire="int8")
    g = synthetic.make_gradients(W, d, "normal", seed=5, device="cuda")
    g[:, 1024:2048] = 0.0
    g[:, 3072:] *= 1e15  # squares stay finite in fp32
    r = gpu_bucketed(gq, g, None, b, cfg)
    assert r["status"] == gq.GQ_OK
    assert r["S"][1] == 0 and r["mult"][1] == 0 and r["unit"][1] == 0
    assert not r["out"][1024:2048].any()
    check(oracle, cfg, g.cpu().numpy(), None, b, r)


def test_nonfinite_bucket_sets_flag(gq):
    W, d, b = 2, 2048, 10
    cfg = gq.GQConfig(s=15, bits=5, wire="int8")
    g = synthetic.make_gradients(W, d, "normal", seed=6, device="cuda")
    g[1, 1500] = float("nan")
    r = gpu_bucketed(gq, g, None, b, cfg)
    assert r["status"] == gq.GQ_ERR_NONFINITE
    assert np.isfinite(r["S"][0]) and np.isnan(r["S"][1])


def test_repeatable(gq):
    W, d, b = 8, 65536, 12
    cfg = gq.GQConfig(s=15, bits=5, wire="int8", seed=17)
    g = synthetic.make_gradients(W, d, "student_t3", seed=3, device="cuda", seg=1000, lo=-4, hi=0)
    a = gpu_bucketed(gq, g, None, b, cfg)
    c = gpu_bucketed(gq, g, None, b, cfg)
    for key in ("S", "codes", "sum", "out"):
        assert np.array_equal(a[key], c[key]), key


def test_host_side_errors(gq):
    cfg = gq.GQConfig(s=15, bits=5, wire="int8")
    with pytest.raises(gq.GQError):
        gq.gq_bucket_count(100, 6)
    with pytest.raises(gq.GQError):
        gq.gq_bucket_count(100, 31)
    flat = torch.zeros(2 * 1000 + 1, dtype=torch.float32, device="cuda")
    g = flat[1:].view(2, 1000)  # contiguous but 4 bytes off a 16-byte boundary
    table = torch.zeros(3 * gq.gq_bucket_count(1000, 7), dtype=torch.float32, device="cuda")
    ws = torch.zeros(gq.gq_bucket_workspace_bytes(cfg, 2, 1000, 7), dtype=torch.uint8,
                     device="cuda")
    with pytest.raises(gq.GQError) as ei:
        gq.gq_bucket_scales(g, None, 7, cfg, table, ws)
    assert ei.value.status == gq.GQ_ERR_ALIGN
    with pytest.raises(gq.GQError) as ei:
        gq.gq_step_bucketed(flat[:2000].view(2, 1000), None, 6, cfg, table, None, None, None, ws)
    assert ei.value.status == gq.GQ_ERR_ARG
