"""Real data-parallel exchange: each rank holds its own workers' gradients.

"Quantize Once, Train Fast: Allreduce-Compatible Compression with Provable
Guarantees" (Abstract): with one global scale shared by all workers, the
quantized gradients are integers on the same grid and can be summed by an
Allreduce.  On one GPU the library simulates that Allreduce by summing W rows;
here each rank runs the same kernels on its own rows and the two exchanges are
real collectives of ``torch.distributed`` (NCCL across GPUs):

1. ``gq_global_norm`` over the rank's rows, then an all-reduce MAX of the one
   fp32 scale;
2. ``gq_quantize_aggregate`` of the rank's rows with that scale (codes drawn as
   workers rank * W_local + w, error feedback applied locally), writing the
   rank's integer sum as int8, or as fp16 holding the integer;
3. an all-reduce SUM of those sums (d or 2d bytes instead of 4d of fp32);
4. ``gq_dequantize_ef`` of the total into the mean over all W = world * W_local
   workers.

Codes, sums and means equal those of the single-GPU path on all W rows given
the same scale; the scale itself is the max of per-rank scales, each within
1e-5 of its fp64 norm.  Packed sub-byte codes cannot be summed by NCCL, so the
exchange carries the unpacked integer sums.  NCCL reduces 8-, 32- and 64-bit
integers but not 16-bit ones, so the exchange takes the int8 wire type (W
times the largest code value at most 127) or the fp16 one (at most 2048: every
partial sum of such integers is an exact fp16 value, in any order); int16
configurations are refused.

With ``chunks > 1`` (one worker per rank) the quantization of chunk k + 1
overlaps the all-reduce of chunk k: each chunk is quantized with
``gq_config.coord0`` set to its first coordinate, so it draws exactly the
uniforms it would draw in the whole vector, and the result is bit-identical
to the unchunked exchange.

``capture(g, e)`` records one whole exchange -- kernels, both NCCL
all-reduces and, when chunked, the overlap between them -- into a CUDA graph,
and ``replay()`` runs it with one host call per step.  The step then comes from
a device word (``gq_config.step_dev``) that the graph itself advances, so
replay k draws exactly the uniforms of step ``first + k``.  The graph is bound
to the addresses of ``g`` and ``e``: write each step's gradients into ``g`` in
place.  ``close()`` releases the graph; call it before the process group is
destroyed.

The library calls are reached through an ``ops`` object (``GpuOps`` by
default) so that the host-side orchestration can be exercised with other
backends in tests; the product path always uses ``GpuOps``.
"""
from dataclasses import replace

import torch
import torch.distributed as dist

from . import (GQ_OK, GQConfig, GQError, gq_advance_step, gq_dequantize_ef,
               gq_get_device_status, gq_global_norm, gq_quantize_aggregate, gq_validate,
               gq_workspace_bytes, gq_workspace_init)


class GpuOps:
    """The library's kernels for one rank's rows."""

    def global_norm(self, g, e, cfg, scale, ws):
        gq_global_norm(g, e, cfg, scale, None, ws)

    def quantize_sum(self, g, e, cfg, scale, sum_out, ws):
        gq_quantize_aggregate(g, e, cfg, scale, None, sum_out, None, ws)

    def decode(self, sum_in, W, cfg, scale, out, ws):
        gq_dequantize_ef(sum_in, None, None, None, W, sum_in.shape[0], cfg, scale, out, ws)

    def status(self, ws):
        return gq_get_device_status(ws)


class DataParallelStep:
    """One compressed gradient exchange per call, for this rank's W_local rows.

    cfg: the quantizer (its ``worker0`` is set per rank); d: coordinates;
    w_local: workers held by each rank (the same on every rank).  The overflow
    rule is checked for the total W = world * w_local."""

    def __init__(self, cfg: GQConfig, d: int, w_local: int = 1, group=None, device=None,
                 ops=None, chunks: int = 1):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.w_local = int(w_local)
        self.W = self.world * self.w_local
        self.d = int(d)
        rc = gq_validate(cfg, self.W, self.d)
        if rc != GQ_OK:
            raise GQError(rc, "DataParallelStep")
        if cfg.wire_dtype not in (torch.int8, torch.float16):
            raise ValueError("NCCL has no 16-bit integer reduction: use wire='int8' (W * max "
                             "code value <= 127) or wire='f16' (<= 2048)")
        self.chunks = max(1, int(chunks))
        if self.chunks > 1 and self.w_local != 1:
            raise ValueError("chunked exchange: one worker per rank (the rows of a chunk must "
                             "be contiguous)")
        # chunk boundaries on 128-coordinate blocks (keeps every chunk's sum,
        # mean and gradient pointers 16-byte aligned)
        step_c = -(-self.d // (self.chunks * 128)) * 128 if self.chunks > 1 else self.d
        self.bounds = [(c0, min(self.d, c0 + step_c)) for c0 in range(0, self.d, max(1, step_c))]
        self.cfg = replace(cfg, worker0=self.rank * self.w_local)
        self.ops = ops if ops is not None else GpuOps()
        dev = torch.device(device) if device is not None else torch.device("cuda")
        self.scale = torch.zeros(1, dtype=torch.float32, device=dev)
        self.sum = torch.zeros(self.d, dtype=cfg.wire_dtype, device=dev)
        self.out = torch.zeros(self.d, dtype=torch.float32, device=dev)
        self.ws = torch.zeros(gq_workspace_bytes(cfg, self.w_local, self.d), dtype=torch.uint8,
                              device=dev)
        if dev.type == "cuda":
            gq_workspace_init(self.ws)
        self.graph = None
        self.step_dev = None

    def _exchange(self, g, e, cfg):
        ef = e if cfg.ef else None
        self.ops.global_norm(g, ef, cfg, self.scale, self.ws)
        dist.all_reduce(self.scale, op=dist.ReduceOp.MAX, group=self.group)
        if self.chunks == 1:
            self.ops.quantize_sum(g, e, cfg, self.scale, self.sum, self.ws)
            dist.all_reduce(self.sum, op=dist.ReduceOp.SUM, group=self.group)
            self.ops.decode(self.sum, self.W, cfg, self.scale, self.out, self.ws)
        else:
            # quantize chunk k + 1 while the all-reduce of chunk k runs on the
            # collective's own stream; decode each chunk once its sum is in
            works = []
            for c0, c1 in self.bounds:
                cfg_k = replace(cfg, coord0=c0)
                self.ops.quantize_sum(g[:, c0:c1], None if e is None else e[:, c0:c1], cfg_k,
                                      self.scale, self.sum[c0:c1], self.ws)
                works.append(dist.all_reduce(self.sum[c0:c1], op=dist.ReduceOp.SUM,
                                             group=self.group, async_op=True))
            for (c0, c1), work in zip(self.bounds, works):
                work.wait()
                self.ops.decode(self.sum[c0:c1], self.W, cfg, self.scale,
                                self.out[c0:c1], self.ws)

    def _check(self):
        rc = self.ops.status(self.ws)
        if rc != GQ_OK:
            raise GQError(rc, "DataParallelStep")

    def __call__(self, g, e=None, step=None, check=False):
        """g: [w_local][d] fp32 on this rank; e: the rank's error rows (updated in
        place when cfg.ef).  Returns the mean over all W workers, [d] fp32."""
        if step is not None:
            self.cfg.step = int(step)
        self._exchange(g, e, self.cfg)
        if check:
            self._check()
        return self.out

    def capture(self, g, e=None, first_step=0):
        """Record one exchange on g (and e) into a CUDA graph; replay() runs it.
        Every rank must capture at the same point, since the graph holds
        collectives.  An eager warm-up on a copy of e first sets each kernel's
        launch attributes and opens the NCCL communicator, leaving e as it was."""
        import torch
        self.close()
        self.step_dev = torch.full((1,), int(first_step), dtype=torch.int32,
                                   device=self.out.device)
        cfg = replace(self.cfg, step_dev=self.step_dev)
        e_warm = None if e is None else e.clone()
        self._exchange(g, e_warm, cfg)
        torch.cuda.synchronize()
        self.step_dev.fill_(int(first_step))
        del e_warm
        graph = torch.cuda.CUDAGraph()
        # thread-local: a CUDA call from the collective library's own threads
        # during the capture does not invalidate it
        with torch.cuda.graph(graph, capture_error_mode="thread_local"):
            self._exchange(g, e, cfg)
            gq_advance_step(self.step_dev)
        self.graph = graph

    def replay(self, step=None, check=False):
        """Run the captured exchange once (the step advances by one per replay;
        `step` sets it first).  Returns the mean over all W workers."""
        if self.graph is None:
            raise RuntimeError("DataParallelStep.replay: nothing captured")
        if step is not None:
            self.step_dev.fill_(int(step))
        self.graph.replay()
        if check:
            self._check()
        return self.out

    def close(self):
        """Release the captured graph (before destroying the process group)."""
        self.graph = None


def gather_rows(local, out, group=None):
    """All-gather each rank's [w_local][n] rows into out [world * w_local][n],
    rank-major, so that row i of out is global worker i."""
    world = dist.get_world_size(group)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(out, local, group=group)
    else:
        dist.all_gather(list(out.chunk(world)), local, group=group)


class DataParallelLqsgdStep:
    """LQ-SGD ("Trustworthy Efficient Communication for Distributed Learning
    using LQ-SGD Algorithm", review, "What carries the argument": P and Q
    log-quantized before they are exchanged, error fed back) with each rank
    holding W_local workers' matrices.

    Log codes are not additive, so the exchange of a factor is an all-gather of
    every worker's int8 codes and per-matrix max-abs values; every rank then
    decodes and sums all W workers in ascending worker order, exactly as the
    single-GPU step does, so P_hat, Q and Ghat are the same on every rank and
    equal the single-GPU step's.  Per step: gq_psgd_project (local) ->
    gq_logq_quantize (local, worker offset) -> all-gather -> gq_logq_decode_sum
    -> gq_psgd_orthonormalize -> gq_psgd_back_project (local) ->
    gq_logq_quantize -> all-gather -> gq_logq_decode_sum -> gq_psgd_mean ->
    gq_psgd_reconstruct."""

    def __init__(self, shapes, w_local=1, alpha=10.0, seed=0, group=None, device=None):
        from . import gq_psgd_workspace_bytes
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.sh = shapes
        self.w_local = int(w_local)
        self.W = self.world * self.w_local
        self.alpha, self.seed = float(alpha), int(seed)
        dev = torch.device(device) if device is not None else torch.device("cuda")
        sh, wl, W = shapes, self.w_local, self.W
        f32, i8 = torch.float32, torch.int8
        self.pw = torch.empty((wl, sh.ptotal), dtype=f32, device=dev)
        self.qw = torch.empty((wl, sh.qtotal), dtype=f32, device=dev)
        self.codes_p_l = torch.empty((wl, sh.ptotal), dtype=i8, device=dev)
        self.codes_q_l = torch.empty((wl, sh.qtotal), dtype=i8, device=dev)
        self.max_p_l = torch.empty((wl, sh.nmats), dtype=f32, device=dev)
        self.max_q_l = torch.empty((wl, sh.nmats), dtype=f32, device=dev)
        self.codes_p = torch.empty((W, sh.ptotal), dtype=i8, device=dev)
        self.codes_q = torch.empty((W, sh.qtotal), dtype=i8, device=dev)
        self.max_p = torch.empty((W, sh.nmats), dtype=f32, device=dev)
        self.max_q = torch.empty((W, sh.nmats), dtype=f32, device=dev)
        self.qsum = torch.empty(sh.qtotal, dtype=f32, device=dev)
        self.ws = torch.zeros(gq_psgd_workspace_bytes(wl, sh), dtype=torch.uint8, device=dev)
        if dev.type == "cuda":
            gq_workspace_init(self.ws)
        self.ranks = [sh.rank] * sh.nmats

    def __call__(self, g, m, p, q, ghat, have_prev, step, check=False):
        """g, m: this rank's [w_local][sum n m] rows (m is the state, updated);
        p, q: P_hat and the mean Q (the same on every rank, updated); ghat:
        [sum n m] output, or None."""
        from . import (gq_logq_decode_sum, gq_logq_quantize, gq_psgd_back_project,
                       gq_psgd_mean, gq_psgd_orthonormalize, gq_psgd_project,
                       gq_psgd_reconstruct)
        sh = self.sh
        cfg = GQConfig(levels="log", alpha=self.alpha, seed=self.seed, step=2 * int(step),
                       worker0=self.rank * self.w_local)
        gq_psgd_project(g, m, sh, have_prev, p, q, self.pw)
        gq_logq_quantize(self.pw, sh.rows, self.ranks, cfg, self.max_p_l, self.codes_p_l, self.ws)
        gather_rows(self.codes_p_l, self.codes_p, self.group)
        gather_rows(self.max_p_l, self.max_p, self.group)
        gq_logq_decode_sum(self.codes_p, self.max_p, sh.rows, self.ranks, cfg, p)
        gq_psgd_orthonormalize(p, sh)
        gq_psgd_back_project(m, p, sh, self.qw, self.ws)
        cfg.step = 2 * int(step) + 1
        gq_logq_quantize(self.qw, sh.cols, self.ranks, cfg, self.max_q_l, self.codes_q_l, self.ws)
        gather_rows(self.codes_q_l, self.codes_q, self.group)
        gather_rows(self.max_q_l, self.max_q, self.group)
        gq_logq_decode_sum(self.codes_q, self.max_q, sh.cols, self.ranks, cfg, self.qsum)
        gq_psgd_mean(self.qsum, q, self.W)
        if ghat is not None:
            gq_psgd_reconstruct(p, q, sh, ghat)
        if check:
            rc = gq_get_device_status(self.ws)
            if rc != GQ_OK:
                raise GQError(rc, "DataParallelLqsgdStep")
        return ghat


class GpuNatOps:
    """The library's natural-compression kernels."""

    def quantize(self, x, cfg, codes, ws):
        from . import gq_nat_quantize
        gq_nat_quantize(x, cfg, codes, ws)

    def decode_sum(self, codes, out):
        from . import gq_nat_decode_sum
        gq_nat_decode_sum(codes, out)

    def status(self, ws):
        return gq_get_device_status(ws)


class DataParallelNatStep:
    """Natural compression (Horvath et al., "Natural Compression for Distributed
    Deep Learning", cited in the Global-QSGD record) across ranks.  Each rank
    rounds its own W_local rows to signed powers of two (gq_nat_quantize, workers
    rank * W_local + w); every coordinate's result is the fp32 sum of all W
    workers' decoded values in ascending worker order, the same on every rank
    and equal to the single-GPU sum.  Powers of two over the whole exponent range
    cannot be summed as fixed-width integers, so the codes travel instead:

    - gather (default): the 16-bit codes are all-gathered (as bytes, rank-major)
      and every rank decodes the whole sum: (N - 1) * 2n bytes in per rank;
    - sharded (one worker per rank): an all-to-all sends each rank the codes of
      its column shard, it decodes and sums that shard, and the fp32 shard sums
      are all-gathered: (N - 1)/N * 6n bytes, against (N - 1)/N * 8n for a ring
      fp32 all-reduce.  Shards are rounded up to 8 coordinates (padding columns
      carry code 0, value 0).

    The kernels are reached through ``ops`` (``GpuNatOps`` by default) so that
    the host orchestration can be tested with other backends."""

    def __init__(self, n, w_local=1, seed=0, group=None, device=None, sharded=False, ops=None):
        from . import gq_workspace_init as _init
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.n = int(n)
        self.w_local = int(w_local)
        self.W = self.world * self.w_local
        self.seed = int(seed)
        self.sharded = bool(sharded)
        self.ops = ops if ops is not None else GpuNatOps()
        dev = torch.device(device) if device is not None else torch.device("cuda")
        if self.sharded:
            if self.w_local != 1:
                raise ValueError("sharded exchange: one worker per rank")
            shard = -(-self.n // self.world)
            self.shard = -(-shard // 8) * 8
            # padded row [N][shard] rank-major; the padding stays code 0
            self.codes_row = torch.zeros((1, self.world * self.shard), dtype=torch.int16,
                                         device=dev)
            self.codes_l = self.codes_row[:, :self.n]
            self.recv = torch.empty((self.world, self.shard), dtype=torch.int16, device=dev)
            self.part = torch.empty(self.shard, dtype=torch.float32, device=dev)
            self.full = torch.empty(self.world * self.shard, dtype=torch.float32, device=dev)
            self.out = self.full[:self.n]
        else:
            self.codes_l = torch.empty((self.w_local, self.n), dtype=torch.int16, device=dev)
            self.codes = torch.empty((self.W, self.n), dtype=torch.int16, device=dev)
            self.out = torch.empty(self.n, dtype=torch.float32, device=dev)
        self.ws = torch.zeros(256, dtype=torch.uint8, device=dev)
        if dev.type == "cuda":
            _init(self.ws)

    def __call__(self, x, step, check=False):
        """x: this rank's [w_local][n] fp32 rows.  Returns the sum over all W
        workers' compressed rows, [n] fp32 (divide by W for the mean)."""
        cfg = GQConfig(levels="nat", seed=self.seed, step=int(step),
                       worker0=self.rank * self.w_local)
        self.ops.quantize(x, cfg, self.codes_l, self.ws)
        if self.sharded:
            dist.all_to_all_single(self.recv.view(torch.uint8).view(-1),
                                   self.codes_row.view(torch.uint8).view(-1), group=self.group)
            self.ops.decode_sum(self.recv, self.part)
            gather_rows(self.part.view(1, -1), self.full.view(self.world, -1), self.group)
        else:
            gather_rows(self.codes_l.view(torch.uint8), self.codes.view(torch.uint8),
                        self.group)
            self.ops.decode_sum(self.codes, self.out)
        if check:
            rc = self.ops.status(self.ws)
            if rc != GQ_OK:
                raise GQError(rc, "DataParallelNatStep")
        return self.out
