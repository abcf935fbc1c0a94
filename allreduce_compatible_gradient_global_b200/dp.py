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

The library calls are reached through an ``ops`` object (``GpuOps`` by
default) so that the host-side orchestration can be exercised with other
backends in tests; the product path always uses ``GpuOps``.
"""
from dataclasses import replace

import torch
import torch.distributed as dist

from . import (GQ_OK, GQConfig, GQError, gq_dequantize_ef, gq_get_device_status,
               gq_global_norm, gq_quantize_aggregate, gq_validate, gq_workspace_bytes,
               gq_workspace_init)


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
                 ops=None):
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

    def __call__(self, g, e=None, step=None, check=False):
        """g: [w_local][d] fp32 on this rank; e: the rank's error rows (updated in
        place when cfg.ef).  Returns the mean over all W workers, [d] fp32."""
        if step is not None:
            self.cfg.step = int(step)
        ef = e if self.cfg.ef else None
        self.ops.global_norm(g, ef, self.cfg, self.scale, self.ws)
        dist.all_reduce(self.scale, op=dist.ReduceOp.MAX, group=self.group)
        self.ops.quantize_sum(g, e, self.cfg, self.scale, self.sum, self.ws)
        dist.all_reduce(self.sum, op=dist.ReduceOp.SUM, group=self.group)
        self.ops.decode(self.sum, self.W, self.cfg, self.scale, self.out, self.ws)
        if check:
            rc = self.ops.status(self.ws)
            if rc != GQ_OK:
                raise GQError(rc, "DataParallelStep")
        return self.out
