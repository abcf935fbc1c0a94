"""Stream order under the dependent launch.  The norm and fused passes may be
scheduled before the kernel ahead of them in the stream has finished; each
waits for it before touching global memory.  These tests issue work with no
host synchronization between the calls and compare it, bit for bit, with the
same work synchronized after every call:

- a torch kernel writes the gradient, then the step runs at once (the norm
  pass follows a kernel that never signals its dependents);
- error-feedback steps run back to back with nothing between them (each
  norm pass reads the error rows the previous fused pass wrote, and each fused
  pass the scale its norm pass wrote);
- a torch kernel reads the mean right after the fused pass.
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


def run_steps(gq, cfg, src, T, sync, write_g):
    """T steps; write_g: a torch kernel rewrites the gradient before each step
    (else it is written once, and each norm pass directly follows the previous
    step's fused pass)."""
    W, d = src.shape
    buf = gq.StepBuffers(cfg, W, d)
    g = torch.zeros_like(src)
    g.copy_(src)
    outs, scales = [], []
    for t in range(T):
        cfg.step = t
        if write_g:
            g.copy_(src)      # a torch kernel writes the gradient ...
            g.mul_(1.0 + t)
        if sync:
            torch.cuda.synchronize()
        gq.gq_step_fused(g, buf.e, cfg, buf.scale, buf.norms, buf.codes, buf.sum, buf.out,
                         buf.ws)  # ... and the step follows it at once
        if sync:
            torch.cuda.synchronize()
        if write_g:  # a torch kernel reads the mean at once
            outs.append(buf.out.clone())
            scales.append(buf.scale.clone())
    if not write_g:  # nothing between the steps: the last step's results only
        outs.append(buf.out.clone())
        scales.append(buf.scale.clone())
    torch.cuda.synchronize()
    assert gq.gq_get_device_status(buf.ws) == gq.GQ_OK
    return outs, scales, (buf.e.clone() if buf.e is not None else None), buf.codes.clone()


@pytest.mark.parametrize("W,d,kw", [
    (8, 1 << 18, dict(s=15, bits=5, wire="int8", ef=True)),
    (4, 1 << 20, dict(s=15, bits=5, wire="int8")),
    (8, 300_000, dict(levels="exp", L=8, bits=5, wire="int16", scale_kind="maxabs", ef=True)),
    (8, 1 << 23, dict(s=127, bits=8, wire="int16", ef=True)),
])
@pytest.mark.parametrize("write_g", [True, False])
def test_unsynchronized_steps_equal_synchronized_steps(gq, W, d, kw, write_g):
    src = synthetic.make_gradients(W, d, "normal_seg", seed=W + d, device="cuda", seg=4096,
                                   lo=-3, hi=0)
    a = run_steps(gq, gq.GQConfig(seed=21, **kw), src, 5, sync=False, write_g=write_g)
    b = run_steps(gq, gq.GQConfig(seed=21, **kw), src, 5, sync=True, write_g=write_g)
    assert len(a[0]) == len(b[0]) == (5 if write_g else 1)
    for t in range(len(a[0])):
        assert torch.equal(a[0][t].view(torch.int32), b[0][t].view(torch.int32)), t
        assert torch.equal(a[1][t], b[1][t]), t
    if kw.get("ef"):
        assert torch.equal(a[2].view(torch.int32), b[2].view(torch.int32))
    assert torch.equal(a[3], b[3])
