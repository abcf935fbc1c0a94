"""gq_global_norm_noalloc: the global-scale call for callers that cannot
allocate device memory (another allocator owns the device, or the path cannot
afford cudaMalloc and its device-wide synchronization).  It keeps its partial
sums in a fixed array inside the library instead of a caller workspace.

Checked through the C ABI on two calls in a row (the second finds the shared
scratch as the first left it):

* against the ordinary gq_global_norm bit for bit -- both run the same kernel
  with the same block count, so the scale and the per-worker norms agree
  exactly;
* against the oracle's fp64 norm (the tolerance the other scale tests use:
  1e-5 relative for L2, exact for max-abs), so a drift of the shared norm
  kernel away from the oracle fails here too;
* and that the second call changes neither the device's free memory nor
  torch's allocated bytes (the first call may load the module and resolve the
  array's address).

This file is collected last, so a run that stops at the first failure has run
every other test before it.
"""
import ctypes
import gc

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


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def call_noalloc(gq, g, e, cfg, scale, norms):
    c = cfg.c()
    W, d = g.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return gq.lib().gq_global_norm_noalloc(_p(g), _p(e), W, d, ctypes.byref(c), _p(scale),
                                           _p(norms), stream)


@pytest.mark.parametrize("W,d,kind,ef", [
    (4, 1 << 20, "l2", False),
    (8, 25_557_032 // 16, "l2", False),
    (8, 100_003, "maxabs", False),       # scalar-load rows
    (3, 77_777, "l2", True),
    (1, 4096, "maxabs", True),
    (64, 5000, "l2", False),
])
def test_noalloc_matches_workspace_form_and_oracle(gq, oracle, W, d, kind, ef):
    cfg = gq.GQConfig(s=15, bits=5, wire="int8", scale_kind=kind, ef=ef)
    g = synthetic.make_gradients(W, d, "student_t3", seed=W + d, device="cuda", seg=4096,
                                 lo=-4, hi=0)
    e = (synthetic.make_gradients(W, d, "normal", seed=d, device="cuda") * 1e-3) if ef else None
    ref = gq.StepBuffers(cfg, W, d)
    gq.gq_global_norm(g, e, cfg, ref.scale, ref.norms, ref.ws)
    torch.cuda.synchronize()
    S_ref, n_ref = ref.scale.item(), ref.norms.cpu().numpy()
    S_ora, n_ora = oracle.global_scale(g.cpu().numpy(), None if e is None else e.cpu().numpy(),
                                       0 if kind == "l2" else 1)
    for call in range(2):
        scale = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
        norms = torch.full((W,), -1.0, dtype=torch.float64, device="cuda")
        torch.cuda.synchronize()
        # no collection of unrelated garbage (tensors of earlier tests) may free
        # memory between the two readings
        gc.collect()
        gc.disable()
        try:
            free0, alloc0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
            assert call_noalloc(gq, g, e, cfg, scale, norms) == gq.GQ_OK
            torch.cuda.synchronize()
            free1, alloc1 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
        finally:
            gc.enable()
        if call == 1:  # the first call may load the module; the second allocates nothing
            assert free1 == free0
            assert alloc1 == alloc0
        S, n = scale.item(), norms.cpu().numpy()
        assert S == S_ref, (call, S, S_ref)
        assert np.array_equal(n.view(np.uint64), n_ref.view(np.uint64)), call
        if kind == "l2":
            assert abs(S - float(S_ora)) <= SCALE_RTOL * float(S_ora), (call, S, S_ora)
            assert np.allclose(n, n_ora, rtol=SCALE_RTOL, atol=0), call
        else:
            assert S == S_ora, (call, S, S_ora)
            assert np.array_equal(n, n_ora), call


def test_noalloc_rejects_sizes_beyond_its_maximum(gq):
    cfg = gq.GQConfig(s=1, bits=4, wire="int16")
    g = torch.zeros((4097, 8), device="cuda")
    scale = torch.zeros(1, device="cuda")
    assert call_noalloc(gq, g, None, cfg, scale, None) == gq.GQ_ERR_SIZE
    # and a zero-size gradient is fine: S = 0
    g0 = torch.zeros((2, 0), device="cuda")
    scale.fill_(5.0)
    assert call_noalloc(gq, g0, None, cfg, scale, None) == gq.GQ_OK
    torch.cuda.synchronize()
    assert scale.item() == 0.0
