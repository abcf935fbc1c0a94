"""The data-parallel exchange on the GPU through NCCL (one rank on this GPU).

With one rank holding all W workers, ``DataParallelStep`` runs the library's
kernels and two real NCCL all-reduces; its mean must equal the single-GPU fused
step's bit for bit (same rows, same partition, so the same scale), and its
error buffers too.  Two or more ranks need two or more GPUs; their host-side
orchestration is covered by tests/test_dp_exchange.py with gloo on CPU.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import synthetic

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.fixture(scope="module")
def gq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import allreduce_compatible_gradient_global_b200 as gq
    return gq


@pytest.mark.parametrize("kw,ef", [(dict(s=15, bits=5, wire="int8"), False),
                                   (dict(levels="exp", L=5, bits=4, wire="int8",
                                         scale_kind="maxabs"), True),
                                   (dict(levels="exp", L=8, bits=5, wire="f16"), False),
                                   (dict(s=127, bits=8, wire="f16"), True)])
def test_nccl_single_rank_equals_fused_step(gq, kw, ef):
    from allreduce_compatible_gradient_global_b200.dp import DataParallelStep
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        W, d = 4, 100_003
        cfg = gq.GQConfig(seed=7, ef=ef, **kw)
        g = synthetic.make_gradients(W, d, "student_t3", seed=1, device="cuda", seg=1000,
                                     lo=-4, hi=0)
        e1 = torch.zeros_like(g)
        e2 = torch.zeros_like(g)
        stepper = DataParallelStep(cfg, d, w_local=W)
        buf = gq.StepBuffers(cfg, W, d, ef=False)
        for t in range(3):
            cfg.step = t
            out = stepper(g, e1, step=t, check=True).clone()
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
