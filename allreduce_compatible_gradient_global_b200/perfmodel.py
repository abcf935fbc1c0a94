"""A bandwidth model of the path, and of the real data-parallel step it stands in for.

"Quantize Once, Train Fast: Allreduce-Compatible Compression with Provable
Guarantees" (Abstract) says a performance model was developed to evaluate the
method across hardware; its content is not given.  This is a plain one:

* On one GPU, each kernel is a launch latency plus its algorithmic bytes over an
  effective HBM bandwidth, both fitted by least squares from measured times
  (``fit_launch_and_bandwidth``).
* In a real data-parallel step each worker is its own GPU.  The compressed step
  is the local norm pass, a scalar MAX all-reduce for the shared scale, the
  local quantize pass, a SUM all-reduce of the int8/int16 codes, and the local
  decode.  The uncompressed step is one fp32 SUM all-reduce.  A ring all-reduce
  of B bytes over N ranks costs alpha + 2 (N - 1) / N * B / link_bandwidth.
* Natural compression (a gather-style compressor) exchanges codes instead of a
  sum: an all-gather of every rank's 2n bytes ((N - 1) * 2n in per rank), or,
  sharded, an all-to-all of code shards ((N - 1)/N * 2n) and an all-gather of
  fp32 shard sums ((N - 1)/N * 4n).

Everything here is host arithmetic on numbers the caller measures or chooses;
nothing runs on the GPU.
"""
from dataclasses import dataclass

import numpy as np


def step_bytes(W, d, bits, sum_bytes, ef=False, row_bytes=None):
    """Algorithmic bytes of (pass 1, pass 2) of one simulated step of W workers.

    Pass 1 reads the gradients (and the error buffers).  Pass 2 reads them
    again, writes the packed codes, the integer sum and the fp32 mean, and with
    error feedback reads and writes the error buffers.  row_bytes defaults to
    the padded wire row: ceil(d / 128) blocks of 16 * bits bytes."""
    if row_bytes is None:
        row_bytes = -(-d // 128) * 16 * bits
    p1 = 4 * W * d * (2 if ef else 1)
    p2 = 4 * W * d + W * row_bytes + sum_bytes * d + 4 * d + (8 * W * d if ef else 0)
    return p1, p2


def fit_launch_and_bandwidth(bytes_moved, seconds):
    """Least-squares fit of seconds = launch + bytes / bandwidth.

    Returns (launch_seconds, bandwidth_bytes_per_second).  Needs at least two
    distinct byte counts."""
    x = np.asarray(bytes_moved, dtype=np.float64)
    y = np.asarray(seconds, dtype=np.float64)
    if x.size < 2 or np.ptp(x) == 0:
        raise ValueError("need at least two distinct sizes")
    A = np.stack([np.ones_like(x), x], axis=1)
    (launch, inv_bw), *_ = np.linalg.lstsq(A, y, rcond=None)
    if inv_bw <= 0:
        raise ValueError("times do not grow with size")
    return float(launch), float(1.0 / inv_bw)


def ring_allreduce_seconds(nbytes, ranks, link_bytes_per_s, alpha_s):
    """alpha + 2 (N - 1) / N * bytes / link bandwidth; zero work for one rank."""
    if ranks <= 1:
        return 0.0
    return alpha_s + 2.0 * (ranks - 1) / ranks * nbytes / link_bytes_per_s


@dataclass
class Machine:
    """Bandwidths in bytes/s, latencies in seconds.  Defaults: the measured B200
    copy bandwidth and NVLink 5 peer bandwidth on this class of machine, and
    latencies of the order an NCCL call and a kernel launch take."""
    hbm: float = 6528.7e9
    link: float = 770e9
    allreduce_alpha: float = 15e-6
    launch: float = 4e-6
    pass2_efficiency: float = 0.81  # measured fraction of hbm the fused pass reaches
    # (5-bit codes, int8 sums, no error feedback, on the ResNet-50-sized workload)


def dp_step_seconds(d, ranks, bits=8, sum_bytes=1, m=Machine(), compressed=True, chunks=1):
    """One data-parallel gradient exchange with one worker per GPU.

    compressed: norm pass + MAX all-reduce of 4 bytes + quantize pass + SUM
    all-reduce of d * sum_bytes + decode pass (read the sum, write the mean).
    Otherwise: a SUM all-reduce of 4 * d bytes.  chunks > 1: the quantize pass
    and the SUM all-reduce run as a K-stage pipeline (chunk k + 1 quantized
    while chunk k is summed), each chunk paying its own launch and alpha."""
    if not compressed:
        return ring_allreduce_seconds(4.0 * d, ranks, m.link, m.allreduce_alpha)
    norm = m.launch + 4.0 * d / m.hbm
    scale = ring_allreduce_seconds(4.0, ranks, m.link, m.allreduce_alpha)
    decode = m.launch + (sum_bytes * d + 4.0 * d) / m.hbm
    K = max(1, int(chunks))
    dk = d / K
    quant = m.launch + (4.0 * dk + dk * bits / 8.0) / (m.hbm * m.pass2_efficiency)
    summ = ring_allreduce_seconds(sum_bytes * dk, ranks, m.link, m.allreduce_alpha)
    # a K-stage two-resource pipeline: first quantize, then the slower of the
    # two stages K - 1 times, then the last all-reduce
    pipelined = quant + (K - 1) * max(quant, summ) + summ
    return norm + scale + pipelined + decode


def crossover_d(ranks, bits=8, sum_bytes=1, m=Machine(), lo=1, hi=1 << 40):
    """Smallest d (bisection over integers) from which the compressed exchange
    is faster than the fp32 all-reduce; None if it never is within [lo, hi]."""
    def gain(d):
        return (dp_step_seconds(d, ranks, bits, sum_bytes, m, compressed=False)
                - dp_step_seconds(d, ranks, bits, sum_bytes, m, compressed=True))
    if gain(hi) <= 0:
        return None
    if gain(lo) > 0:
        return lo
    while hi - lo > 1:
        mid = (lo + hi) // 2
        if gain(mid) > 0:
            hi = mid
        else:
            lo = mid
    return hi


def all_gather_seconds(nbytes_per_rank, ranks, link_bytes_per_s, alpha_s):
    """Ring all-gather of nbytes from every rank: each rank receives the other
    N - 1 contributions, alpha + (N - 1) * bytes / link bandwidth."""
    if ranks <= 1:
        return 0.0
    return alpha_s + (ranks - 1) * nbytes_per_rank / link_bytes_per_s


def all_to_all_seconds(nbytes_per_rank, ranks, link_bytes_per_s, alpha_s):
    """All-to-all of an nbytes buffer split evenly over N ranks: each rank sends
    and receives (N - 1)/N of it, alpha + (N - 1)/N * bytes / link bandwidth."""
    if ranks <= 1:
        return 0.0
    return alpha_s + (ranks - 1) / ranks * nbytes_per_rank / link_bytes_per_s


def nat_step_seconds(n, ranks, m=Machine(), sharded=False, quant_efficiency=0.77,
                     decode_efficiency=0.91):
    """One natural-compression exchange with one worker per GPU: the quantize
    pass (read 4n, write 2n), then either an all-gather of the 2n-byte codes and
    a decode-sum over all N workers (read 2Nn, write 4n), or, sharded, an
    all-to-all of code shards, a decode-sum of this rank's shard (read 2N
    shard, write 4 shard) and an all-gather of the fp32 shard sums.  The two
    efficiencies are the measured fractions of hbm the two kernels reach."""
    N = max(1, int(ranks))
    quant = m.launch + 6.0 * n / (m.hbm * quant_efficiency)
    if not sharded:
        move = all_gather_seconds(2.0 * n, N, m.link, m.allreduce_alpha)
        decode = m.launch + (2.0 * N * n + 4.0 * n) / (m.hbm * decode_efficiency)
        return quant + move + decode
    shard = -(-int(n) // N)
    a2a = all_to_all_seconds(2.0 * N * shard, N, m.link, m.allreduce_alpha)
    decode = m.launch + (2.0 * N * shard + 4.0 * shard) / (m.hbm * decode_efficiency)
    gather = all_gather_seconds(4.0 * shard, N, m.link, m.allreduce_alpha)
    return quant + a2a + decode + gather


def nat_crossover_d(ranks, m=Machine(), sharded=True, lo=1, hi=1 << 40):
    """Smallest n (bisection over integers) from which the natural-compression
    exchange is faster than the fp32 all-reduce; None if it never is in
    [lo, hi]."""
    def gain(n):
        return (dp_step_seconds(n, ranks, m=m, compressed=False)
                - nat_step_seconds(n, ranks, m=m, sharded=sharded))
    if gain(hi) <= 0:
        return None
    if gain(lo) > 0:
        return lo
    while hi - lo > 1:
        mid = (lo + hi) // 2
        if gain(mid) > 0:
            hi = mid
        else:
            lo = mid
    return hi

