"""The data-parallel exchange's host orchestration, on CPU with gloo ranks.

Each rank holds its own rows and runs ``DataParallelStep``; the kernels are
stood in for by the oracle (test-only ``ops``), so what is checked is the
exchange itself: the MAX all-reduce of the scale, worker indices rank * W_local
+ w for the uniforms, the SUM all-reduce of the integer sums, the decode over
all W workers, and local error feedback.  The result must equal the oracle's
single-process step on all W rows, bit for bit (the oracle's per-worker norms do
not depend on how rows are grouped).
"""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import synthetic


class OracleOps:
    """The oracle in place of the kernels, for host-side tests only."""

    def __init__(self, oracle):
        self.o = oracle

    def _kw(self, cfg):
        return dict(levels=0 if cfg.levels == "uniform" else 1, s=cfg.s, L=cfg.L)

    def global_norm(self, g, e, cfg, scale, ws):
        kind = 0 if cfg.scale_kind == "l2" else 1
        S, _ = self.o.global_scale(g.numpy(), None if e is None else e.numpy(), kind)
        scale[0] = float(S)

    def quantize_sum(self, g, e, cfg, scale, sum_out, ws):
        S = np.float32(scale[0].item())
        ev = e.numpy() if (cfg.ef and e is not None) else None
        n = g.shape[1]
        codes = self.o.quantize(g.numpy(), ev, seed=cfg.seed, step=cfg.step, S=S,
                                worker0=cfg.worker0,
                                js=np.arange(cfg.coord0, cfg.coord0 + n, dtype=np.int64),
                                **self._kw(cfg))
        sum_out.copy_(torch.from_numpy(self.o.aggregate(codes, levels=self._kw(cfg)["levels"],
                                                        L=cfg.L)).to(sum_out.dtype))
        if cfg.ef and e is not None:
            e.copy_(torch.from_numpy(self.o.error_feedback(g.numpy(), ev, codes, S=S,
                                                           **self._kw(cfg))))

    def decode(self, sum_in, W, cfg, scale, out, ws):
        S = np.float32(scale[0].item())
        out.copy_(torch.from_numpy(self.o.decode_mean(sum_in.numpy().astype(np.int32), W, S=S,
                                                      **self._kw(cfg))))

    def status(self, ws):
        return 0


def _store(tmp_path):
    """The rendezvous of a test's group: a file store in the test's own
    directory, so no TCP port can collide with another process's."""
    return "file://" + str(tmp_path / "store")


CASES = {
    "uniform": dict(levels="uniform", s=15, bits=5, wire="int8", seed=3, step=2),
    "exp_ef": dict(levels="exp", L=5, bits=4, wire="int8", scale_kind="maxabs", ef=True,
                   seed=5, step=1),
    "exp_f16": dict(levels="exp", L=8, bits=5, wire="f16", seed=6, step=0),
    "u127_f16": dict(s=127, bits=8, wire="f16", ef=True, seed=7, step=3),
}


def _rank_main(rank, world, store, case, w_local, d, outdir, chunks=1):
    import datetime
    dist.init_process_group("gloo", init_method=store, rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        import allreduce_compatible_gradient_global_b200 as gq
        from allreduce_compatible_gradient_global_b200.dp import DataParallelStep
        cfg = gq.GQConfig(**CASES[case])
        W = world * w_local
        g_all = synthetic.make_gradients(W, d, "student_t3", seed=11, seg=100, lo=-3, hi=0)
        e_all = synthetic.make_gradients(W, d, "normal", seed=12) * 1e-3
        rows = slice(rank * w_local, (rank + 1) * w_local)
        g = g_all[rows].clone()
        e = e_all[rows].clone()
        stepper = DataParallelStep(cfg, d, w_local=w_local, device="cpu", ops=OracleOps(oracle),
                                   chunks=chunks)
        outs = []
        for t in range(2):
            outs.append(stepper(g, e, step=cfg.step + t).clone().numpy())
        np.savez(os.path.join(outdir, f"rank{rank}.npz"), out0=outs[0], out1=outs[1],
                 e=e.numpy(), scale=stepper.scale.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("case,w_local,chunks", [("uniform", 1, 1), ("uniform", 3, 1),
                                                  ("exp_ef", 2, 1), ("exp_f16", 2, 1),
                                                  ("u127_f16", 4, 1), ("uniform", 1, 3),
                                                  ("exp_ef", 1, 2)])
def test_two_ranks_equal_the_single_process_step(oracle, tmp_path, case, w_local, chunks):
    """chunks > 1: chunk k + 1 is quantized while chunk k is all-reduced; each
    chunk draws the uniforms of its own coordinates (coord0)."""
    world, d = 2, 700
    mp.start_processes(_rank_main, args=(world, _store(tmp_path), case, w_local, d, str(tmp_path),
                                         chunks),
                       nprocs=world, join=True, start_method="spawn")
    import allreduce_compatible_gradient_global_b200 as gq
    cfg = gq.GQConfig(**CASES[case])
    W = world * w_local
    g_all = synthetic.make_gradients(W, d, "student_t3", seed=11, seg=100, lo=-3, hi=0).numpy()
    e = (synthetic.make_gradients(W, d, "normal", seed=12) * 1e-3).numpy()
    kw = dict(levels=0 if cfg.levels == "uniform" else 1, s=cfg.s, L=cfg.L,
              scale_kind=0 if cfg.scale_kind == "l2" else 1)
    res = [np.load(tmp_path / f"rank{r}.npz") for r in range(world)]
    for t in range(2):
        ref = oracle.step(g_all, e if cfg.ef else None, seed=cfg.seed, step=cfg.step + t,
                          ef=cfg.ef, **kw)
        for r in range(world):
            got = res[r][f"out{t}"]
            assert np.array_equal(got.view(np.uint32), ref["out"].view(np.uint32)), (t, r)
        if cfg.ef:
            e = ref["e"]
    if cfg.ef:
        for r in range(world):
            rows = slice(r * w_local, (r + 1) * w_local)
            assert np.array_equal(res[r]["e"].view(np.uint32), e[rows].view(np.uint32))
    assert res[0]["scale"][0] == res[1]["scale"][0]


def test_overflow_rule_uses_the_total_worker_count(oracle):
    """W = world * W_local decides the wire type: 9 workers of s = 15 overflow int8;
    the fp16 sums hold integers up to 2048."""
    import allreduce_compatible_gradient_global_b200 as gq
    assert gq.gq_validate(gq.GQConfig(s=15, bits=5, wire="int8"), 8, 100) == gq.GQ_OK
    assert gq.gq_validate(gq.GQConfig(s=15, bits=5, wire="int8"), 9, 100) == gq.GQ_ERR_OVERFLOW
    assert gq.gq_validate(gq.GQConfig(s=127, bits=8, wire="f16"), 16, 100) == gq.GQ_OK
    assert gq.gq_validate(gq.GQConfig(s=127, bits=8, wire="f16"), 17, 100) == \
        gq.GQ_ERR_OVERFLOW
    assert gq.gq_validate(gq.GQConfig(levels="exp", L=8, bits=5, wire="f16"), 16, 100) == \
        gq.GQ_OK
    assert gq.gq_validate(gq.GQConfig(levels="exp", L=8, bits=5, wire="f16"), 17, 100) == \
        gq.GQ_ERR_OVERFLOW


def test_worker0_offsets_the_uniform_streams(oracle):
    """Rows quantized as workers k.. equal rows k.. of a quantization of all rows."""
    g = synthetic.make_gradients(5, 300, "normal", seed=2).numpy()
    full = oracle.quantize(g, s=7, seed=9, step=4, S=np.float32(40.0))
    part = oracle.quantize(g[2:4], s=7, seed=9, step=4, S=np.float32(40.0), worker0=2)
    assert np.array_equal(full[2:4], part)
    assert not np.array_equal(full[0:2], part)


def test_int16_wire_is_refused(tmp_path):
    """NCCL cannot reduce 16-bit integers: the exchange refuses int16 sums up front."""
    import allreduce_compatible_gradient_global_b200 as gq
    from allreduce_compatible_gradient_global_b200.dp import DataParallelStep
    dist.init_process_group("gloo", init_method=_store(tmp_path), rank=0, world_size=1)
    try:
        with pytest.raises(ValueError):
            DataParallelStep(gq.GQConfig(s=127, bits=8, wire="int16"), 100, device="cpu")
    finally:
        dist.destroy_process_group()


def _gather_main(rank, world, store, outdir):
    dist.init_process_group("gloo", init_method=store, rank=rank, world_size=world)
    try:
        import oracle
        from allreduce_compatible_gradient_global_b200.dp import gather_rows
        w_local, sizes = 2, np.array([300, 120], np.int64)
        W = world * w_local
        x = synthetic.make_gradients(W, int(sizes.sum()), "normal", seed=4).numpy()
        rows = slice(rank * w_local, (rank + 1) * w_local)
        mx_l, codes_l = oracle.logq_quantize(x[rows], sizes, seed=9, step=2,
                                             worker0=rank * w_local)
        codes = torch.empty((W, int(sizes.sum())), dtype=torch.int8)
        mx = torch.empty((W, sizes.size), dtype=torch.float32)
        gather_rows(torch.from_numpy(codes_l), codes)
        gather_rows(torch.from_numpy(mx_l), mx)
        total = oracle.logq_decode_sum(codes.numpy(), mx.numpy(), sizes)
        np.save(os.path.join(outdir, f"lq{rank}.npy"), total)
    finally:
        dist.destroy_process_group()


def test_gathered_log_codes_decode_like_one_process(oracle, tmp_path):
    """Each rank log-quantizes its own workers (worker offset rank * W_local),
    the codes and max-abs values are all-gathered rank-major, and every rank's
    decoded sum equals the single-process decode of all workers, bit for bit."""
    world = 2
    mp.start_processes(_gather_main, args=(world, _store(tmp_path), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    sizes = np.array([300, 120], np.int64)
    x = synthetic.make_gradients(4, int(sizes.sum()), "normal", seed=4).numpy()
    mx, codes = oracle.logq_quantize(x, sizes, seed=9, step=2)
    ref = oracle.logq_decode_sum(codes, mx, sizes)
    for r in range(world):
        got = np.load(tmp_path / f"lq{r}.npy")
        assert np.array_equal(got.view(np.uint32), ref.view(np.uint32)), r


class OracleNatOps:
    """The oracle in place of the natural-compression kernels (host tests only)."""

    def __init__(self, oracle):
        self.o = oracle

    def quantize(self, x, cfg, codes, ws):
        c = self.o.nat_quantize(x.numpy(), seed=cfg.seed, step=cfg.step, worker0=cfg.worker0)
        codes.copy_(torch.from_numpy(c.view(np.int16)))

    def decode_sum(self, codes, out):
        out.copy_(torch.from_numpy(self.o.nat_decode_sum(codes.numpy().view(np.uint16))))

    def status(self, ws):
        return 0


def _nat_main(rank, world, store, outdir, w_local, n, sharded):
    dist.init_process_group("gloo", init_method=store, rank=rank, world_size=world)
    try:
        import oracle
        from allreduce_compatible_gradient_global_b200.dp import DataParallelNatStep
        W = world * w_local
        x = synthetic.make_gradients(W, n, "student_t3", seed=6, seg=50, lo=-20, hi=3)
        rows = slice(rank * w_local, (rank + 1) * w_local)
        step = DataParallelNatStep(n, w_local=w_local, seed=4, device="cpu", sharded=sharded,
                                   ops=OracleNatOps(oracle))
        outs = [step(x[rows].clone(), t).clone().numpy() for t in (9, 10)]
        np.savez(os.path.join(outdir, f"nat{rank}.npz"), out0=outs[0], out1=outs[1])
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,w_local,n,sharded", [(2, 2, 301, False), (2, 1, 301, True),
                                                     (3, 1, 1000, True), (3, 1, 5, True)])
def test_natural_exchange_sums_like_one_process(oracle, tmp_path, world, w_local, n, sharded):
    """Gather: each rank compresses its own workers (worker offset rank * W_local)
    and the codes are all-gathered as bytes.  Sharded: an all-to-all hands each
    rank the codes of its column shard, which it decodes and sums, and the fp32
    shard sums are all-gathered.  Either way every rank's sum equals the
    single-process sum of all workers, bit for bit."""
    mp.start_processes(_nat_main,
                       args=(world, _store(tmp_path), str(tmp_path), w_local, n, sharded),
                       nprocs=world, join=True, start_method="spawn")
    W = world * w_local
    x = synthetic.make_gradients(W, n, "student_t3", seed=6, seg=50, lo=-20, hi=3).numpy()
    for t in (9, 10):
        ref = oracle.nat_decode_sum(oracle.nat_quantize(x, seed=4, step=t))
        for r in range(world):
            got = np.load(tmp_path / f"nat{r}.npz")[f"out{t - 9}"]
            assert np.array_equal(got.view(np.uint32), ref.view(np.uint32)), (t, r)


def test_sharded_natural_exchange_needs_one_worker_per_rank(tmp_path):
    """The column shards are slices of one code row: more rows per rank are refused."""
    from allreduce_compatible_gradient_global_b200.dp import DataParallelNatStep
    dist.init_process_group("gloo", init_method=_store(tmp_path), rank=0, world_size=1)
    try:
        with pytest.raises(ValueError):
            DataParallelNatStep(100, w_local=2, device="cpu", sharded=True)
        step = DataParallelNatStep(101, w_local=1, device="cpu", sharded=True)
        assert step.shard % 8 == 0 and step.shard * step.world >= 101
        assert step.codes_l.is_contiguous() and step.codes_l.shape == (1, 101)
    finally:
        dist.destroy_process_group()

