"""Natural compression on the GPU against the oracle.

Codes bit for bit over single coordinates, ragged groups of four, scalar rows
(n % 4 != 0), many grid-stride iterations and a worker offset; the decoded
fp32 sums over workers bit for bit; the device step word; the non-finite flag;
and the ResNet-50-sized launch (8 x 25,557,032) on sampled columns.
"""
import numpy as np
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


def inputs(W, n, seed):
    """Per-segment scales over 35 decades, plus zeros, subnormals and a power of two."""
    x = synthetic.make_gradients(W, n, "student_t3", seed=seed, seg=64, lo=-30, hi=5).numpy()
    if n >= 6:
        x[0, :6] = np.array([0.0, -0.0, 1e-40, -2e-39, 2.0 ** -126, 1.0], np.float32)
    return x


def workspace(gq):
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    gq.gq_workspace_init(ws)
    return ws


def run(gq, x, cfg):
    W, n = x.shape
    xd = torch.from_numpy(x).cuda()
    codes = torch.empty((W, n), dtype=torch.int16, device="cuda")
    out = torch.empty(n, dtype=torch.float32, device="cuda")
    ws = workspace(gq)
    gq.gq_nat_quantize(xd, cfg, codes, ws)
    gq.gq_nat_decode_sum(codes, out)
    assert gq.gq_get_device_status(ws) == gq.GQ_OK
    return codes.cpu().numpy().view(np.uint16), out.cpu().numpy()


@pytest.mark.parametrize("W,n", [(1, 1), (3, 5), (4, 1023), (2, 4099), (8, 4100), (8, 100_003),
                                 (5, 1 << 18), (1, 77)])
def test_codes_and_sums_match_the_oracle(gq, oracle, W, n):
    x = inputs(W, n, seed=n)
    cfg = gq.GQConfig(levels="nat", seed=0xABCDEF0123, step=3, worker0=2)
    got_codes, got_sum = run(gq, x, cfg)
    ref = oracle.nat_quantize(x, seed=0xABCDEF0123, step=3, worker0=2)
    assert np.array_equal(got_codes, ref)
    want = oracle.nat_decode_sum(ref)
    assert np.array_equal(got_sum.view(np.uint32), want.view(np.uint32))


def test_device_step_word_equals_the_host_step(gq):
    x = inputs(4, 10_000, seed=1)
    a, _ = run(gq, x, gq.GQConfig(levels="nat", seed=5, step=41))
    step_dev = torch.full((1,), 41, dtype=torch.int32, device="cuda")
    b, _ = run(gq, x, gq.GQConfig(levels="nat", seed=5, step=0, step_dev=step_dev))
    assert np.array_equal(a, b)
    c, _ = run(gq, x, gq.GQConfig(levels="nat", seed=5, step=42))
    assert not np.array_equal(a, c)


def test_nonfinite_input_raises_the_flag(gq):
    x = torch.ones((2, 64), dtype=torch.float32, device="cuda")
    x[1, 7] = float("inf")
    x[0, 3] = float("nan")
    codes = torch.empty((2, 64), dtype=torch.int16, device="cuda")
    ws = workspace(gq)
    gq.gq_nat_quantize(x, gq.GQConfig(levels="nat"), codes, ws)
    assert gq.gq_get_device_status(ws) == gq.GQ_ERR_NONFINITE
    assert int(codes[1, 7]) == 0xFF
    x[1, 7] = 2.0
    x[0, 3] = -0.5
    gq.gq_nat_quantize(x, gq.GQConfig(levels="nat"), codes, ws)
    assert gq.gq_get_device_status(ws) == gq.GQ_OK  # the flag was cleared by the read


@pytest.mark.parametrize("W,n", [(8, 25_557_032), (3, 5_000_003)])
def test_full_size_launch_on_sampled_columns(gq, oracle, W, n):
    """The bench's launch (and a scalar-row one) checked on 4096 sampled columns
    per row, the first and last columns included."""
    if W == 8:
        x = synthetic.workload_gradients("resnet50_t3_w8", device="cuda")
    else:
        x = synthetic.make_gradients(W, n, "normal", seed=9, device="cuda")
    cfg = gq.GQConfig(levels="nat", seed=77, step=12)
    codes = torch.empty((W, n), dtype=torch.int16, device="cuda")
    out = torch.empty(n, dtype=torch.float32, device="cuda")
    ws = workspace(gq)
    gq.gq_nat_quantize(x, cfg, codes, ws)
    gq.gq_nat_decode_sum(codes, out)
    assert gq.gq_get_device_status(ws) == gq.GQ_OK
    rng = np.random.default_rng(n)
    js = np.unique(np.concatenate([[0, n - 1], rng.integers(0, n, 4094)])).astype(np.int64)
    jt = torch.from_numpy(js).cuda()
    xs = x[:, jt].cpu().numpy()
    ref = oracle.nat_quantize(xs, seed=77, step=12, js=js)
    assert np.array_equal(codes[:, jt].cpu().numpy().view(np.uint16), ref)
    assert np.array_equal(out[jt].cpu().numpy().view(np.uint32),
                          oracle.nat_decode_sum(ref).view(np.uint32))
