"""Seeded synthetic inputs for the tests and the benchmark.

This module holds no quantization arithmetic: it only draws gradients of the
shapes and value distributions of the workloads (the pages train ResNet-18 on
CIFAR/ImageNet; no datasets or trained weights are available, so flattened
gradient vectors with per-segment scales stand in for per-layer gradients).
Both the CUDA path and the oracle consume what it returns; neither produces it.

Recipes (every draw comes from one seeded torch.Generator on the requested
device, workers in ascending order, so a (recipe, seed, step) triple fixes the
data on a given device type):

* ``normal``      N(0, 1).
* ``student_t3``  per segment k of ``seg`` coordinates, sigma_k = 10^U(lo, hi)
                  (shared by all workers: a segment is a layer), entries
                  sigma_k * Z / sqrt(chi2_3 / 3) with Z ~ N(0,1).
* ``laplace``     per segment b_k = 10^U(lo, hi), entries b_k * (E1 - E2) with
                  E1, E2 ~ Exp(1) (a Laplace(0, b_k) draw).
* ``normal_seg``  per segment sigma_k = 10^U(lo, hi), entries sigma_k * N(0,1).
"""
import math

import numpy as np
import torch

MASTER_SEED = 0x51D5EED

# Workload table: name -> generator recipe and the quantizer settings the
# workload is run with.  d and W are the sizes of the gradient vectors.
WORKLOADS = {
    "normal_d2^20_w4": dict(W=4, d=1 << 20, recipe="normal", levels="uniform", s=15,
                            bits=5, wire="int8", scale="l2", ef=False, seed_index=0),
    "resnet50_t3_w8": dict(W=8, d=25_557_032, recipe="student_t3", seg=1 << 17,
                           lo=-4.0, hi=-1.0, levels="uniform", s=15, bits=5,
                           wire="int8", scale="l2", ef=False, seed_index=1),
    "gpt2s_laplace_w8": dict(W=8, d=124_439_808, recipe="laplace", seg=1 << 16,
                             lo=-5.0, hi=-2.0, levels="exp", L=8, bits=5,
                             wire="int16", scale="maxabs", ef=False, seed_index=2),
    # the same gradients with the L2 global scale (the second scale variant)
    "gpt2s_laplace_w8_l2": dict(W=8, d=124_439_808, recipe="laplace", seg=1 << 16,
                                lo=-5.0, hi=-2.0, levels="exp", L=8, bits=5,
                                wire="int16", scale="l2", ef=False, seed_index=2),
    # a fresh draw every step (the step enters the seed), error feedback carried over
    "normal_seg_d2^30_w8_ef": dict(W=8, d=1 << 30, recipe="normal_seg", seg=1 << 20,
                                   lo=-4.0, hi=0.0, levels="uniform", s=127, bits=8,
                                   wire="int16", scale="l2", ef=True, steps=5,
                                   fresh_per_step=True, seed_index=3),
}

# LQ-SGD factor workload: per worker, `pairs` factor pairs P (n x r), Q (m x r).
LQ_WORKLOAD = dict(W=8, pairs=24, n=4096, m=4096, ranks=(1, 4, 7), alpha=10.0,
                   seed_index=4)


def seed_for(seed_index: int, step: int = 0) -> int:
    return MASTER_SEED + seed_index + 1_000_003 * step


def _segment_scales(gen, nseg, lo, hi, device):
    u = torch.rand(nseg, generator=gen, device=device, dtype=torch.float64)
    return torch.pow(10.0, lo + (hi - lo) * u).to(torch.float32)


def fill_gradients(out: torch.Tensor, recipe: str, seed: int, seg: int = 0,
                   lo: float = 0.0, hi: float = 0.0) -> torch.Tensor:
    """Fill ``out`` ([W][d] float32, any device) in place with the recipe."""
    assert out.dtype == torch.float32 and out.dim() == 2
    W, d = out.shape
    device = out.device
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    if recipe == "normal":
        for w in range(W):
            out[w].normal_(generator=gen)
        return out
    nseg = max(1, math.ceil(d / seg))
    scales = _segment_scales(gen, nseg, lo, hi, device)
    nfull = d // seg

    def scale_row(row):
        # multiply segment k by its scale without a per-coordinate temporary
        if nfull:
            row[: nfull * seg].view(nfull, seg).mul_(scales[:nfull, None])
        if nfull * seg < d:
            row[nfull * seg:].mul_(scales[nfull])

    for w in range(W):
        row = out[w]
        if recipe == "normal_seg":
            row.normal_(generator=gen)
        elif recipe == "student_t3":
            row.normal_(generator=gen)
            chi = torch.empty_like(row)
            acc = torch.zeros_like(row)
            for _ in range(3):
                chi.normal_(generator=gen)
                acc.addcmul_(chi, chi)
            del chi
            row.div_(torch.sqrt(acc.div_(3.0)))
            del acc
        elif recipe == "laplace":
            row.exponential_(generator=gen)
            e2 = torch.empty_like(row).exponential_(generator=gen)
            row.sub_(e2)
            del e2
        else:
            raise ValueError(f"unknown recipe {recipe}")
        scale_row(row)
    return out


def make_gradients(W: int, d: int, recipe: str = "normal", seed: int = MASTER_SEED,
                   device="cpu", seg: int = 0, lo: float = 0.0, hi: float = 0.0,
                   out: torch.Tensor = None) -> torch.Tensor:
    if out is None:
        out = torch.empty((W, d), dtype=torch.float32, device=device)
    return fill_gradients(out, recipe, seed, seg, lo, hi)


def workload_gradients(name: str, device="cpu", step: int = 0, out=None, W=None, d=None):
    """Gradients of a named workload (optionally truncated to W workers / d coords:
    the truncated draw is a different sample of the same distribution)."""
    wl = WORKLOADS[name]
    W = W or wl["W"]
    d = d or wl["d"]
    return make_gradients(W, d, wl["recipe"], seed_for(wl["seed_index"], step), device,
                          wl.get("seg", 0), wl.get("lo", 0.0), wl.get("hi", 0.0), out)


def lq_sizes(rank: int, pairs: int = 24, n: int = 4096, m: int = 4096):
    """Element counts of the 2*pairs factor matrices of one worker: P_0, Q_0, P_1, ..."""
    sizes = []
    for _ in range(pairs):
        sizes += [n * rank, m * rank]
    return np.asarray(sizes, dtype=np.int64)


def lq_factors(rank: int, W: int = 8, pairs: int = 24, seed: int = None, device="cpu"):
    """[W][sum(sizes)] float32 of N(0,1) factor entries, plus the sizes."""
    sizes = lq_sizes(rank, pairs)
    seed = seed_for(LQ_WORKLOAD["seed_index"]) + rank if seed is None else seed
    x = make_gradients(W, int(sizes.sum()), "normal", seed, device)
    return x, sizes


def numpy_normal(W, d, seed):
    """Small CPU-only draws for oracle property tests."""
    return np.random.default_rng(seed).standard_normal((W, d)).astype(np.float32)
