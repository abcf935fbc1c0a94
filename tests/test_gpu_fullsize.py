"""Full-size workloads on the GPU, in the launch configuration the benchmark
times (gq_global_norm + gq_quantize_aggregate writing packed codes, the sum
and the mean), checked against the oracle on sampled 128-coordinate blocks.

Sampling is sound because every code depends only on (S, seed, step, worker,
coordinate, v): once the scale is known, any subset of coordinates can be
checked on its own.  The scale itself is checked at full size against the
oracle's fp64 sum of squares (or max-abs), streamed through host memory in
chunks in one ascending pass.
"""
import numpy as np
import pytest
import torch

import synthetic

pytestmark = pytest.mark.gpu

CHUNK = 1 << 26  # floats per host chunk of the streamed scale check


@pytest.fixture(scope="module")
def gq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import allreduce_compatible_gradient_global_b200 as gq
    return gq


def config_of(gq, wl, **over):
    kw = dict(levels=wl["levels"], s=wl.get("s", 15), L=wl.get("L", 8), bits=wl["bits"],
              scale_kind=wl["scale"], wire=wl["wire"], ef=wl["ef"], seed=0xC0FFEE, step=0)
    kw.update(over)
    return gq.GQConfig(**kw)


def streamed_scale(oracle, g, e, kind):
    """Oracle scale of device tensors g (and e), one row at a time in chunks."""
    W, d = g.shape
    norms = np.zeros(W)
    hg = torch.empty(min(CHUNK, d), dtype=torch.float32).pin_memory()
    he = torch.empty(min(CHUNK, d), dtype=torch.float32).pin_memory() if e is not None else None
    for w in range(W):
        acc = 0.0
        mx = np.float32(0)
        for j in range(0, d, CHUNK):
            n = min(CHUNK, d - j)
            hg[:n].copy_(g[w, j:j + n])
            if e is not None:
                he[:n].copy_(e[w, j:j + n])
            gn = hg[:n].numpy()
            en = he[:n].numpy() if e is not None else None
            if kind == "l2":
                acc = oracle.sumsq_from(acc, gn, en)
            else:
                mx = max(mx, oracle.maxabs(gn, en))
        norms[w] = np.sqrt(acc) if kind == "l2" else float(mx)
    return np.float32(norms.max()), norms


def sampled_blocks(d, n, seed):
    nblk = (d + 127) // 128
    rng = np.random.default_rng(seed)
    picks = set(rng.integers(0, nblk, size=n).tolist()) | {0, nblk - 1}
    return sorted(picks)


def check_blocks(gq, oracle, cfg, g, e_before, buf, e_after, blocks):
    W, d = g.shape
    kw = dict(levels=0 if cfg.levels == "uniform" else 1, s=cfg.s, L=cfg.L)
    S = np.float32(buf.scale.item())
    bb = 16 * cfg.bits
    codes_gpu = buf.codes.view(W, -1, bb)
    for b in blocks:
        j0, j1 = 128 * b, min(128 * b + 128, d)
        js = np.arange(j0, j1, dtype=np.int64)
        gs = g[:, j0:j1].cpu().numpy()
        es = e_before[:, j0:j1].cpu().numpy() if e_before is not None else None
        codes = oracle.quantize(gs, es, seed=cfg.seed, step=cfg.step, S=S, js=js, **kw)
        packed = oracle.pack(codes, cfg.bits)
        assert np.array_equal(codes_gpu[:, b, :].cpu().numpy(), packed), f"codes, block {b}"
        total = oracle.aggregate(codes, levels=kw["levels"], L=cfg.L)
        assert np.array_equal(buf.sum[j0:j1].cpu().numpy().astype(np.int32), total), b
        out = oracle.decode_mean(total, W, S=S, **kw)
        assert np.array_equal(buf.out[j0:j1].cpu().numpy().view(np.uint32), out.view(np.uint32)), b
        if e_after is not None:
            e_ref = oracle.error_feedback(gs, es, codes, S=S, **kw)
            assert np.array_equal(e_after[:, j0:j1].cpu().numpy().view(np.uint32),
                                  e_ref.view(np.uint32)), b


def run_bench_launches(gq, g, e, cfg, buf):
    gq.gq_global_norm(g, e if cfg.ef else None, cfg, buf.scale, buf.norms, buf.ws)
    gq.gq_quantize_aggregate(g, e, cfg, buf.scale, buf.codes, buf.sum, buf.out, buf.ws)
    assert gq.gq_get_device_status(buf.ws) == gq.GQ_OK


@pytest.mark.parametrize("name,over", [
    ("resnet50_t3_w8", {}),
    ("resnet50_t3_w8", dict(bits=8)),
    ("gpt2s_laplace_w8", {}),
    ("gpt2s_laplace_w8", dict(scale_kind="l2")),
    ("normal_d2^20_w4", {}),
])
def test_full_size_workload(gq, oracle, name, over):
    wl = synthetic.WORKLOADS[name]
    cfg = config_of(gq, wl, **over)
    g = synthetic.workload_gradients(name, device="cuda")
    W, d = g.shape
    buf = gq.StepBuffers(cfg, W, d)
    run_bench_launches(gq, g, None, cfg, buf)
    S_ref, norms_ref = streamed_scale(oracle, g, None, cfg.scale_kind)
    S = np.float32(buf.scale.item())
    if cfg.scale_kind == "l2":
        assert abs(float(S) - float(S_ref)) <= 1e-5 * float(S_ref)
        assert np.allclose(buf.norms.cpu().numpy(), norms_ref, rtol=1e-5)
    else:
        assert S == S_ref
    check_blocks(gq, oracle, cfg, g, None, buf, None, sampled_blocks(d, 48, 1))
    del g, buf
    torch.cuda.empty_cache()


def test_d2_30_error_feedback_five_steps(gq, oracle):
    name = "normal_seg_d2^30_w8_ef"
    wl = synthetic.WORKLOADS[name]
    W, d = wl["W"], wl["d"]
    cfg = config_of(gq, wl)
    g = torch.empty((W, d), dtype=torch.float32, device="cuda")
    buf = gq.StepBuffers(cfg, W, d)        # e starts at zero
    blocks = sampled_blocks(d, 24, 2)
    for t in range(wl["steps"]):
        cfg.step = t
        synthetic.workload_gradients(name, device="cuda", step=t, out=g)
        e_before = {b: buf.e[:, 128 * b:128 * b + 128].clone() for b in blocks}
        S_ref, _ = streamed_scale(oracle, g, buf.e, "l2")
        run_bench_launches(gq, g, buf.e, cfg, buf)
        S = np.float32(buf.scale.item())
        assert abs(float(S) - float(S_ref)) <= 1e-5 * float(S_ref), t
        for b in blocks:
            check_blocks_one(gq, oracle, cfg, g[:, 128 * b:128 * b + 128], e_before[b], buf, b)
    del g, buf
    torch.cuda.empty_cache()


def check_blocks_one(gq, oracle, cfg, gs, es, buf, b):
    """One 128-coordinate block of the d = 2^30 step (a multiple of 128)."""
    W = gs.shape[0]
    kw = dict(levels=0, s=cfg.s, L=cfg.L)
    S = np.float32(buf.scale.item())
    j0 = 128 * b
    js = np.arange(j0, j0 + 128, dtype=np.int64)
    gh, eh = gs.cpu().numpy(), es.cpu().numpy()
    codes = oracle.quantize(gh, eh, seed=cfg.seed, step=cfg.step, S=S, js=js, **kw)
    bb = 16 * cfg.bits
    got = buf.codes.view(W, -1, bb)[:, b, :].cpu().numpy()
    assert np.array_equal(got, oracle.pack(codes, cfg.bits)), b
    total = oracle.aggregate(codes)
    assert np.array_equal(buf.sum[j0:j0 + 128].cpu().numpy().astype(np.int32), total), b
    out = oracle.decode_mean(total, W, S=S, **kw)
    assert np.array_equal(buf.out[j0:j0 + 128].cpu().numpy().view(np.uint32), out.view(np.uint32))
    e_ref = oracle.error_feedback(gh, eh, codes, S=S, **kw)
    assert np.array_equal(buf.e[:, j0:j0 + 128].cpu().numpy().view(np.uint32),
                          e_ref.view(np.uint32)), b


@pytest.mark.parametrize("b", [12, 17])
def test_full_size_bucketed(gq, oracle, b):
    """The benchmark workload with one scale per bucket of 2^b coordinates:
    sampled whole buckets (first, last (ragged) and a few between) against the
    oracle's bucket composition on the bucket's coordinates alone."""
    name = "resnet50_t3_w8"
    wl = synthetic.WORKLOADS[name]
    cfg = config_of(gq, wl)
    g = synthetic.workload_gradients(name, device="cuda")
    W, d = g.shape
    nk = gq.gq_bucket_count(d, b)
    table = torch.empty(3 * nk, dtype=torch.float32, device="cuda")
    ws = torch.empty(gq.gq_bucket_workspace_bytes(cfg, W, d, b), dtype=torch.uint8,
                     device="cuda")
    gq.gq_workspace_init(ws)
    buf = gq.StepBuffers(cfg, W, d)
    gq.gq_step_bucketed(g, None, b, cfg, table, buf.codes, buf.sum, buf.out, ws)
    assert gq.gq_get_device_status(ws) == gq.GQ_OK
    t = table.cpu().numpy()
    kw = dict(levels=0 if cfg.levels == "uniform" else 1, s=cfg.s, L=cfg.L,
              scale_kind=0 if cfg.scale_kind == "l2" else 1)
    rng = np.random.default_rng(b)
    picks = sorted(set(rng.integers(0, nk, size=4).tolist()) | {0, nk - 1})
    B = 1 << b
    bb = 16 * cfg.bits
    codes_gpu = buf.codes.view(W, -1, bb)
    for k in picks:
        j0, j1 = k * B, min(d, (k + 1) * B)
        gs = g[:, j0:j1].cpu().numpy()
        S_k = t[k]
        ref_S = oracle.step_bucketed(gs, bucket=B, bits=None, **kw)["S"][0]
        if kw["scale_kind"] == 0:
            assert abs(float(S_k) - float(ref_S)) <= 1e-5 * float(ref_S), k
        else:
            assert S_k == ref_S, k
        codes = oracle.quantize(gs, seed=cfg.seed, step=cfg.step, S=S_k,
                                js=np.arange(j0, j1, dtype=np.int64),
                                levels=kw["levels"], s=cfg.s, L=cfg.L)
        blk0, blk1 = j0 // 128, -(-j1 // 128)
        packed = oracle.pack(codes, cfg.bits)
        got = codes_gpu[:, blk0:blk1, :].cpu().numpy().reshape(W, -1)
        if not np.array_equal(got, packed):
            mine = oracle.unpack(got, W, j1 - j0, cfg.bits)
            w, j = np.nonzero(mine != codes)
            raise AssertionError(
                f"bucket {k}: {w.size} codes differ; S_k={S_k!r} a_k={t[nk + k]!r} "
                f"oracle a={oracle.uniform_multiplier(cfg.s, S_k)!r}; first (w, j, v, gpu, "
                f"oracle): {[(int(a), int(b) + j0, float(gs[a, b]), int(mine[a, b]), int(codes[a, b])) for a, b in zip(w[:6], j[:6])]}")
        total = oracle.aggregate(codes, levels=kw["levels"], L=cfg.L)
        assert np.array_equal(buf.sum[j0:j1].cpu().numpy().astype(np.int32), total), k
        out = oracle.decode_mean(total, W, levels=kw["levels"], s=cfg.s, L=cfg.L, S=S_k)
        assert np.array_equal(buf.out[j0:j1].cpu().numpy().view(np.uint32), out.view(np.uint32))
    del g, buf, table, ws
    torch.cuda.empty_cache()


def test_beyond_2_31_coordinates(gq, oracle):
    """One worker with d = 2^31 + 4 (8.6 GB of gradient): coordinate indices
    pass 2^31, so a 32-bit index anywhere would show.  The scale is checked
    against the oracle's streamed fp64 norm, and sampled blocks on both sides
    of 2^31 (and the last one) bit for bit."""
    W, d = 1, (1 << 31) + 4
    cfg = gq.GQConfig(levels="uniform", s=15, bits=5, wire="int8", seed=77, step=1)
    g = torch.empty((W, d), dtype=torch.float32, device="cuda")
    synthetic.fill_gradients(g, "normal", seed=31)
    buf = gq.StepBuffers(cfg, W, d)
    run_bench_launches(gq, g, None, cfg, buf)
    S_ref, _ = streamed_scale(oracle, g, None, "l2")
    S = np.float32(buf.scale.item())
    assert abs(float(S) - float(S_ref)) <= 1e-5 * float(S_ref)
    nblk = (d + 127) // 128
    edge = (1 << 31) // 128  # the last block: coordinates 2^31 .. 2^31 + 3
    assert edge == nblk - 1
    blocks = sorted({0, 12345, edge - 3, edge - 2, edge - 1, edge})
    check_blocks(gq, oracle, cfg, g, None, buf, None, blocks)
    del g, buf
    torch.cuda.empty_cache()
