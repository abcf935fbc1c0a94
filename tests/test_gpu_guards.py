"""Out-of-bounds writes and checkpoint/resume, on the GPU.

Guard bands: every buffer a call writes is carved out of a larger allocation
whose 4 KiB before and after are filled with a byte pattern; after the call the
bands must be untouched.  This stands in for a memory checker (which is not
available on this pool) at the shapes most likely to go wrong: ragged blocks,
d % 4 != 0 (scalar rows), single coordinates, ragged buckets and row chunks.

Checkpoint / resume: the state of a step is (seed, step, buffers); the
uniforms are counter-based, so 2 steps, a save of the state to host memory, a
restore into fresh buffers and 3 more steps equal 5 uninterrupted steps bit
for bit.
"""
import numpy as np
import pytest
import torch

import synthetic

pytestmark = pytest.mark.gpu

GUARD = 4096
PATTERN = 0xA5


@pytest.fixture(scope="module")
def gq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import allreduce_compatible_gradient_global_b200 as gq
    return gq


class Guarded:
    """Buffers with guard bands on both sides."""

    def __init__(self):
        self.flats = []

    def make(self, shape, dtype, fill=None):
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        flat = torch.full((GUARD + n + GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
        view = flat[GUARD:GUARD + n].view(dtype).view(*shape)
        if fill is not None:
            view.copy_(fill)
        self.flats.append(flat)
        return view

    def check(self):
        torch.cuda.synchronize()
        for i, f in enumerate(self.flats):
            head, tail = f[:GUARD], f[-GUARD:]
            assert bool((head == PATTERN).all()) and bool((tail == PATTERN).all()), \
                f"guard band of buffer {i} overwritten"


STEP_CASES = [
    (3, 1, dict(s=15, bits=5, wire="int8", ef=True)),
    (4, 129, dict(s=15, bits=5, wire="int8")),
    (8, 4099, dict(s=127, bits=8, wire="int16", ef=True)),
    (8, 65536 + 44, dict(s=15, bits=5, wire="int8", ef=True)),
    (8, 40002, dict(levels="exp", L=8, bits=5, wire="int16", scale_kind="maxabs")),
    (5, 7777, dict(s=1000, bits=16, wire="int16")),
    (40, 1028, dict(s=3, bits=4, wire="int8")),
]


@pytest.mark.parametrize("W,d,kw", STEP_CASES)
def test_step_and_split_calls_stay_in_bounds(gq, W, d, kw):
    cfg = gq.GQConfig(seed=1, **kw)
    G = Guarded()
    g = G.make((W, d), torch.float32,
               synthetic.make_gradients(W, d, "student_t3", seed=d, device="cuda", seg=100,
                                        lo=-3, hi=0))
    e = G.make((W, d), torch.float32, torch.zeros((W, d), device="cuda")) if cfg.ef else None
    scale = G.make((1,), torch.float32)
    norms = G.make((W,), torch.float64)
    codes = G.make((W, gq.gq_packed_row_bytes(cfg, d)), torch.uint8)
    sum_ = G.make((d,), cfg.wire_dtype)
    out = G.make((d,), torch.float32)
    ws = G.make((gq.gq_workspace_bytes(cfg, W, d),), torch.uint8, torch.zeros(1, device="cuda"))
    gq.gq_workspace_init(ws)
    gq.gq_step_fused(g, e, cfg, scale, norms, codes, sum_, out, ws)
    assert gq.gq_get_device_status(ws) == gq.GQ_OK
    G.check()
    gq.gq_quantize_pack(g, e, cfg, scale, codes, ws)
    gq.gq_aggregate(codes, W, d, cfg, sum_, ws)
    gq.gq_dequantize_ef(sum_, codes, g, e, W, d, cfg, scale, out, ws)
    G.check()


@pytest.mark.parametrize("W,d,b", [(3, 777, 7), (4, 10001, 10), (2, 3 * 8192 + 1000, 13)])
def test_bucketed_calls_stay_in_bounds(gq, W, d, b):
    cfg = gq.GQConfig(s=15, bits=5, wire="int8", ef=True, seed=2)
    G = Guarded()
    g = G.make((W, d), torch.float32, synthetic.make_gradients(W, d, "normal", seed=b,
                                                               device="cuda"))
    e = G.make((W, d), torch.float32, torch.zeros((W, d), device="cuda"))
    nk = gq.gq_bucket_count(d, b)
    table = G.make((3 * nk,), torch.float32)
    codes = G.make((W, gq.gq_packed_row_bytes(cfg, d)), torch.uint8)
    sum_ = G.make((d,), torch.int8)
    out = G.make((d,), torch.float32)
    ws = G.make((gq.gq_bucket_workspace_bytes(cfg, W, d, b),), torch.uint8,
                torch.zeros(1, device="cuda"))
    gq.gq_workspace_init(ws)
    gq.gq_step_bucketed(g, e, b, cfg, table, codes, sum_, out, ws)
    assert gq.gq_get_device_status(ws) == gq.GQ_OK
    G.check()


@pytest.mark.parametrize("W,rows,cols,r", [(2, [37, 1], [20, 8], 3), (3, [200], [1028], 7),
                                           (2, [16] * 66, [12] * 66, 2)])
def test_psgd_calls_stay_in_bounds(gq, W, rows, cols, r):
    sh = gq.PsgdShapes(rows, cols, r)
    G = Guarded()
    g = G.make((W, sh.total), torch.float32,
               synthetic.make_gradients(W, sh.total, "normal", seed=r, device="cuda"))
    m = G.make((W, sh.total), torch.float32, torch.zeros((W, sh.total), device="cuda"))
    p = G.make((sh.ptotal,), torch.float32, torch.zeros(sh.ptotal, device="cuda"))
    q = G.make((sh.qtotal,), torch.float32,
               synthetic.make_gradients(1, sh.qtotal, "normal", seed=9, device="cuda")[0])
    ghat = G.make((sh.total,), torch.float32)
    ws = G.make((gq.gq_psgd_workspace_bytes(W, sh),), torch.uint8, torch.zeros(1, device="cuda"))
    gq.gq_workspace_init(ws)
    for t in range(2):
        gq.gq_lqsgd_step(g, m, sh, t > 0, gq.GQConfig(levels="log", alpha=10.0, seed=3, step=t),
                         p, q, ghat, ws)
    assert gq.gq_get_device_status(ws) == gq.GQ_OK
    G.check()


def test_fused_step_resumes_bit_exactly(gq):
    W, d = 8, 100_000
    cfg = gq.GQConfig(s=127, bits=8, wire="int16", ef=True, seed=99)

    def grads(t):
        return synthetic.make_gradients(W, d, "normal", seed=1000 + t, device="cuda")

    a = gq.StepBuffers(cfg, W, d)
    outs = []
    for t in range(5):
        cfg.step = t
        gq.gq_step_fused(grads(t), a.e, cfg, a.scale, a.norms, a.codes, a.sum, a.out, a.ws)
        outs.append((a.codes.clone(), a.out.clone()))
    b = gq.StepBuffers(cfg, W, d)
    for t in range(2):
        cfg.step = t
        gq.gq_step_fused(grads(t), b.e, cfg, b.scale, b.norms, b.codes, b.sum, b.out, b.ws)
    saved = (cfg.seed, cfg.step, b.e.cpu().numpy().copy())
    del b
    c = gq.StepBuffers(cfg, W, d)
    c.e.copy_(torch.from_numpy(saved[2]))
    for t in range(saved[1] + 1, 5):
        cfg.step = t
        gq.gq_step_fused(grads(t), c.e, cfg, c.scale, c.norms, c.codes, c.sum, c.out, c.ws)
        assert torch.equal(c.codes, outs[t][0]) and torch.equal(c.out, outs[t][1]), t
    assert torch.equal(c.e, a.e)


def test_lqsgd_step_resumes_bit_exactly(gq):
    W, r = 4, 3
    sh = gq.PsgdShapes([128, 64], [96, 64], r)

    def grads(t):
        return synthetic.make_gradients(W, sh.total, "normal", seed=2000 + t, device="cuda")

    def fresh():
        m = torch.zeros((W, sh.total), dtype=torch.float32, device="cuda")
        p = torch.zeros(sh.ptotal, dtype=torch.float32, device="cuda")
        q = synthetic.make_gradients(1, sh.qtotal, "normal", seed=5, device="cuda")[0]
        ghat = torch.empty(sh.total, dtype=torch.float32, device="cuda")
        ws = torch.empty(gq.gq_psgd_workspace_bytes(W, sh), dtype=torch.uint8, device="cuda")
        gq.gq_workspace_init(ws)
        return m, p, q, ghat, ws

    def run(state, t):
        m, p, q, ghat, ws = state
        gq.gq_lqsgd_step(grads(t), m, sh, t > 0, gq.GQConfig(levels="log", alpha=10.0, seed=8,
                                                             step=t), p, q, ghat, ws)
        return ghat.clone()

    full = fresh()
    ref = [run(full, t) for t in range(5)]
    part = fresh()
    for t in range(2):
        run(part, t)
    saved = [x.cpu().numpy().copy() for x in part[:3]]  # m, p, q
    del part
    resumed = fresh()
    for dst, src in zip(resumed[:3], saved):
        dst.copy_(torch.from_numpy(src))
    for t in range(2, 5):
        assert torch.equal(run(resumed, t), ref[t]), t
    for x, y in zip(resumed[:3], full[:3]):
        assert torch.equal(x, y)
