"""The benchmark's multi-rank logic on CPU: world_size 2 over gloo.

Each rank is an independent replica (the path is one GPU's work; there is no
collective on the data path).  The job's time is the max over ranks of each
rank's own device-timed elapsed time, and the value counts every rank's bytes.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = [3.0, 5.0][rank]                 # rank 1 is the slow one
        t = bench.job_time_ms(mine, world, "cpu")
        v = bench.job_gbs(4 * 8 * 1000, 10, t, world)
        q.put((rank, t, v))
    finally:
        dist.destroy_process_group()


def test_job_time_is_max_over_ranks_and_value_sums_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, t, v in got:
        assert t == 5.0
        # 2 ranks x 32000 bytes x 10 steps over 5 ms
        assert abs(v - 2 * 32000 * 10 / 5e-3 / 1e9) < 1e-12


def _fit_main(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import bench
    # rank 1 sees less free host memory (another rank pinned first): the ranks
    # must still agree, or one would skip the collectives the other enters
    avail = [100 << 30, 40 << 30][rank]
    bench.host_available_bytes = lambda: avail
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        fits_big, _ = bench.host_buffers_fit(60 << 30, world, "cpu")
        fits_small, _ = bench.host_buffers_fit(10 << 30, world, "cpu")
        q.put((rank, fits_big, fits_small))
    finally:
        dist.destroy_process_group()


def test_host_buffer_decision_is_the_same_on_every_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_fit_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    # 60 GiB fits rank 0's 80 GiB budget but not rank 1's 32 GiB: both skip;
    # 10 GiB fits both
    assert got == [(0, False, True), (1, False, True)]


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.job_time_ms(7.5, 1, "cpu") == 7.5


def _run_reference(rank):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--steps", "1", "--warmup", "3", "--reference-coords", "4096",
                           "--workload", "normal_d2^20_w4"],
                          capture_output=True, text=True, env=env, timeout=600)


def test_reference_arm_runs_on_rank0_only():
    other = _run_reference(1)
    assert other.returncode == 0 and other.stdout.strip() == ""
    lead = _run_reference(0)
    assert lead.returncode == 0, lead.stderr
    line = json.loads(lead.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
