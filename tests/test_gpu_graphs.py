"""The step captured in a CUDA graph and replayed.

With ``GQConfig.step_dev`` the kernels read the step from a device word, and
``gq_advance_step`` advances it inside the graph; replaying the captured step
(norm pass, fused pass, counter increment) five times must give exactly the
codes, sums, means and error buffers of five eager steps with steps 0..4.
"""
import pytest
import torch

import synthetic

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import allreduce_compatible_gradient_global_b200 as gq
    return gq


@pytest.mark.parametrize("W,d,kw", [(8, 1 << 20, dict(s=15, bits=5, wire="int8")),
                                    (4, 100_003, dict(s=127, bits=8, wire="int16", ef=True)),
                                    (8, 65536, dict(levels="exp", L=8, bits=5, wire="f16"))])
def test_graph_replay_equals_eager_steps(gq, W, d, kw):
    g = synthetic.make_gradients(W, d, "student_t3", seed=d, device="cuda", seg=1000, lo=-4,
                                 hi=0)
    cfg = gq.GQConfig(seed=3, **kw)
    eager = gq.StepBuffers(cfg, W, d)
    ref = []
    for t in range(5):
        cfg.step = t
        gq.gq_step_fused(g, eager.e, cfg, eager.scale, eager.norms, eager.codes, eager.sum,
                         eager.out, eager.ws)
        ref.append([x.clone() for x in (eager.codes, eager.sum, eager.out)] +
                   ([eager.e.clone()] if cfg.ef else []))
    step_dev = torch.zeros(1, dtype=torch.int32, device="cuda")
    gcfg = gq.GQConfig(seed=3, step=12345, step_dev=step_dev, **kw)  # `step` is ignored
    b = gq.StepBuffers(gcfg, W, d)
    # one eager call sets every launch attribute before capture, then back to step 0
    gq.gq_step_fused(g, b.e, gcfg, b.scale, b.norms, b.codes, b.sum, b.out, b.ws)
    torch.cuda.synchronize()
    if b.e is not None:
        b.e.zero_()
    step_dev.zero_()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        gq.gq_step_fused(g, b.e, gcfg, b.scale, b.norms, b.codes, b.sum, b.out, b.ws)
        gq.gq_advance_step(step_dev)
    for t in range(5):
        graph.replay()
        torch.cuda.synchronize()
        got = [b.codes, b.sum, b.out] + ([b.e] if gcfg.ef else [])
        for x, y in zip(got, ref[t]):
            assert torch.equal(x, y), t
    assert int(step_dev.item()) == 5
    assert gq.gq_get_device_status(b.ws) == gq.GQ_OK
    del graph
