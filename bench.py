"""Benchmark of the quantize + aggregate path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-cpu-baseline] [--no-e2e] [--no-extras]

One step = one pass of the whole path over one batch of W synthetic worker
gradients resident in HBM: gq_global_norm (read 1) then gq_quantize_aggregate
(read 2: Philox uniforms, stochastic rounding, packed codes at wire width,
integer sum over workers, decoded mean, error feedback).  These two calls are
exactly what gq_step_fused issues; the benchmark makes them separately so that
CUDA events can bracket each kernel.

The default workload is the largest one-GPU configuration: W = 8 workers of
d = 2^30 coordinates, per-2^20-segment sigma_k * N(0,1) gradients, uniform
levels s = 127, 8-bit codes, int16 sums, error feedback.  Every step draws a
fresh gradient (the step enters the seed) while the error buffers carry over.
Each step is timed by its own CUDA events around the two kernels; the next
step's gradient is drawn between the timed spans.  A step moves ~174 GiB of
algorithmic bytes, so the events cost nothing measurable, and the 32 GiB
gradient far exceeds L2.  Other workloads (--workload) have fixed gradients:
K steps back to back with events around the run only, and the per-kernel
launch times from K further steps with an event around each kernel (an event
between two kernels drains the GPU at the boundary).

Metric: fp32 gradient GB/s = 4 * W * d bytes / step time (whole job: summed
over ranks under torchrun, each rank an independent replica, timed as the max
over ranks).  Prints one JSON line on rank 0 with the roofline of the dominant
kernel, an end-to-end figure through host buffers (gq_step_fused_host), the CPU
oracle single- and multi-threaded, and, at one GPU, the other workloads under
"configs" (value, roofline and CPU oracle for each).

Other modes print their own JSON line: --sweep (d = 2^16..2^30, EF off/on,
eager and graph-replayed, oracle beside each row), --buckets (per-bucket
scales), --lq (the log quantizer), --lqsgd (the PowerSGD + LQ step), --nat
(natural compression), --dp (the real exchange under torchrun, eager and
graph-replayed, against an fp32 all-reduce).

--impl reference times the CPU oracle (the plain restatement of the method
used by the tests) on the host cores, on a bounded sample of the same
workload, with the same metric.
"""
import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synthetic  # noqa: E402

METRIC = "quantize+aggregate fp32-gradient GB/s at 1 B200; % of HBM roofline"
DEFAULT_WORKLOAD = "normal_seg_d2^30_w8_ef"
# the workload of the extension modes (--buckets, --nat, --dp) unless --workload says otherwise
MODE_WORKLOAD = "resnet50_t3_w8"
# the other configurations, reported under "configs" in the one-GPU line
EXTRA_WORKLOADS = ("normal_d2^20_w4", "resnet50_t3_w8", "gpt2s_laplace_w8", "gpt2s_laplace_w8_l2")
# host oracle samples: a prefix of this many coordinates (None: the whole workload)
CPU_SAMPLE_COORDS = {"normal_seg_d2^30_w8_ef": 1 << 26, "gpt2s_laplace_w8": 1 << 24,
                     "gpt2s_laplace_w8_l2": 1 << 24}
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 1024 * 1024
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "quant_kernel_traffic.json")
KERNEL_SOURCES = ["allreduce_compatible_gradient_global_b200/csrc/gq_quant_tma.cu",
                  "allreduce_compatible_gradient_global_b200/csrc/gq_kernels.cu",
                  "allreduce_compatible_gradient_global_b200/csrc/gq_device.cuh",
                  "allreduce_compatible_gradient_global_b200/csrc/gq_internal.h",
                  "allreduce_compatible_gradient_global_b200/csrc/gq_pdl.cuh"]
LOGQ_SOURCES = ["allreduce_compatible_gradient_global_b200/csrc/gq_logq.cu",
                "allreduce_compatible_gradient_global_b200/csrc/gq_device.cuh",
                "allreduce_compatible_gradient_global_b200/csrc/gq_internal.h"]
LOGQ_COUNTS_FILE = os.path.join(ROOT, "profiles", "logq_kernel_counts.json")
# Issue peak of the log quantizer's roofline: every SM's four schedulers issue
# one warp instruction (32 thread instructions) per clock at the maximum SM clock.
SM_COUNT_B200 = 148
ISSUE_PER_SM_PER_CLK = 4 * 32


def source_hash(files=KERNEL_SOURCES):
    h = hashlib.sha256()
    for rel in files:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def kernel_source_hash():
    return source_hash(KERNEL_SOURCES)


def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def recorded_traffic(workload, d):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary, if it was taken on the current kernel source; else None.  A
    capture of a smaller case of the same recipe (captured_d coordinates) is
    scaled to d: every byte the kernel moves is proportional to d."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    if rec.get("source_hash") != kernel_source_hash():
        return None
    ent = rec.get("workloads", {}).get(workload)
    if ent is None:
        return None
    return float(ent["dram_bytes_per_launch"]) * d / float(ent.get("captured_d", d))


# ----------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML in a thread."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, device_index):
        self.samples = []
        self.times = []        # time.perf_counter() of each sample
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            uuid = None
            try:
                uuid = torch.cuda.get_device_properties(device_index).uuid
            except Exception:
                uuid = None
            handle = None
            if uuid is not None:
                try:
                    handle = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + str(uuid)).encode())
                except Exception:
                    handle = None
            if handle is None:
                vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
                phys = int(vis.split(",")[device_index]) if vis and vis.split(",")[0].isdigit() \
                    else device_index
                handle = pynvml.nvmlDeviceGetHandleByIndex(phys)
            self.handle = handle
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM)
        except Exception as exc:  # no NVML: report that instead of clocks
            self.nvml = None
            self.error = f"nvml unavailable: {exc}"

    def _run(self):
        nv = self.nvml
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                self.samples.append(mhz)
                self.times.append(time.perf_counter())
                self.reasons |= int(rs)
            except Exception:
                pass
            self._stop.wait(0.002)

    def start(self):
        if self.nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()

    def median_between(self, t0, t1):
        """Median SM clock of the samples taken in [t0, t1] (perf_counter
        seconds), or None if none fell there."""
        m = [c for t, c in zip(self.times, self.samples) if t0 <= t <= t1]
        return statistics.median(m) if m else None

    def summary(self):
        if self.nvml is None:
            return {"error": self.error}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


# ------------------------------------------------------------------------ runs
def workload_config(gq, name):
    wl = synthetic.WORKLOADS[name]
    cfg = gq.GQConfig(levels=wl["levels"], s=wl.get("s", 15), L=wl.get("L", 8), bits=wl["bits"],
                      scale_kind=wl["scale"], wire=wl["wire"], ef=wl["ef"], seed=0x5EED, step=0)
    return wl, cfg


def oracle_kwargs(wl):
    return dict(levels=0 if wl["levels"] == "uniform" else 1, s=wl.get("s", 15),
                L=wl.get("L", 8), scale_kind=0 if wl["scale"] == "l2" else 1, bits=wl["bits"],
                seed=0x5EED)


def algorithmic_bytes(gq, cfg, W, d):
    """(pass-1 bytes, pass-2 bytes) per step: what each kernel must move.
    Pass 1 reads g (and e); pass 2 reads g (and e), writes the packed codes,
    the integer sum and the mean (and e)."""
    wire = 1 if cfg.wire == "int8" else 2
    p1 = 4 * W * d + (4 * W * d if cfg.ef else 0)
    p2 = (4 * W * d + W * gq.gq_packed_row_bytes(cfg, d) + wire * d + 4 * d
          + (8 * W * d if cfg.ef else 0))
    return p1, p2


def job_time_ms(elapsed_ms, world, device):
    """The job's time: the max over ranks of each rank's device-timed elapsed ms."""
    if world == 1:
        return float(elapsed_ms)
    t = torch.tensor([float(elapsed_ms)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_gbs(bytes_per_rank_step, steps, job_ms, world):
    """Whole-job throughput: every rank's bytes over the job's (max) time."""
    return world * bytes_per_rank_step * steps / (job_ms * 1e-3) / 1e9


def _sync(world):
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()


def _events(n):
    return [torch.cuda.Event(enable_timing=True) for _ in range(n)]


class Workload:
    """A workload's gradients and step buffers on the device, and its step."""

    def __init__(self, gq, name, dev, d=None):
        self.gq, self.name = gq, name
        self.wl, self.cfg = workload_config(gq, name)
        self.W, self.d = self.wl["W"], (d or self.wl["d"])
        self.fresh = bool(self.wl.get("fresh_per_step", False))
        self.dev = dev
        self.g = synthetic.workload_gradients(name, device=dev, d=self.d)
        self.buf = gq.StepBuffers(self.cfg, self.W, self.d, device=dev)
        self.stream = torch.cuda.current_stream()
        self.drawn = 0  # the step whose gradient g holds

    def draw(self, i):
        """The gradient of step i (fresh-per-step workloads only)."""
        if self.fresh and i != self.drawn:
            synthetic.workload_gradients(self.name, device=self.dev, step=i, out=self.g,
                                         d=self.d)
            self.drawn = i

    def step(self, i, ev=None, codes=True):
        """One step.  ev: two events (around the step) or three (around each
        kernel too; an event between the kernels keeps the fused pass from
        being scheduled before the norm pass ends)."""
        gq, cfg, buf, st = self.gq, self.cfg, self.buf, self.stream
        cfg.step = i
        if ev is not None:
            ev[0].record(st)
        gq.gq_global_norm(self.g, buf.e if cfg.ef else None, cfg, buf.scale, buf.norms, buf.ws,
                          st)
        if ev is not None and len(ev) == 3:
            ev[1].record(st)
        gq.gq_quantize_aggregate(self.g, buf.e, cfg, buf.scale, buf.codes if codes else None,
                                 buf.sum, buf.out, buf.ws, st)
        if ev is not None:
            ev[-1].record(st)

    def check(self, what):
        if self.gq.gq_get_device_status(self.buf.ws, self.stream) != self.gq.GQ_OK:
            raise RuntimeError(f"device flag raised in {what} ({self.name})")

    def free(self):
        del self.g, self.buf
        torch.cuda.empty_cache()


def time_workload(wk, K, warmup, world, flush=None):
    """Times K steps of a workload.  Returns (job ms over the K steps, per-step
    norm ms, per-step fused ms, timing note).  Fresh-per-step workloads and
    those given `flush` (run untimed between steps) are timed step by step;
    the others run K steps back to back, then K more with per-kernel events."""
    dev = wk.dev
    between = None
    if wk.fresh:
        def between(i):
            wk.draw(i)
    elif flush is not None:
        def between(i):
            flush()
    for i in range(warmup):
        if between is not None:
            between(i)
        wk.step(i)
    wk.check("warm-up")
    if between is not None:
        spans_ev = [_events(2) for _ in range(K)]
        _sync(world)
        for i in range(K):
            between(warmup + i)
            wk.step(warmup + i, spans_ev[i])
        _sync(world)
        spans = [e[0].elapsed_time(e[1]) for e in spans_ev]
        job_ms = job_time_ms(sum(spans), world, dev)
        evs = [_events(3) for _ in range(K)]
        for i in range(K):
            between(warmup + K + i)
            wk.step(warmup + K + i, evs[i])
        torch.cuda.synchronize()
        note = ("value, ms_per_step: each step timed by CUDA events around its two kernels; "
                + ("the next step's fresh gradient is drawn between the timed spans"
                   if wk.fresh else "L2 flushed between the timed spans")
                + "; roofline avg_launch_ms: K further steps with events around each kernel")
    else:
        t0, t1 = _events(2)
        _sync(world)
        t0.record(wk.stream)
        for i in range(K):
            wk.step(warmup + i)
        t1.record(wk.stream)
        _sync(world)
        job_ms = job_time_ms(t0.elapsed_time(t1), world, dev)
        evs = [_events(3) for _ in range(K)]
        for i in range(K):
            wk.step(warmup + K + i, evs[i])
        torch.cuda.synchronize()
        note = ("value, ms_per_step: K steps back to back, CUDA events around the whole run "
                "only; roofline avg_launch_ms: K further steps with events around each kernel")
    wk.check("timed steps")
    norm_ms = [e[0].elapsed_time(e[1]) for e in evs]
    quant_ms = [e[1].elapsed_time(e[2]) for e in evs]
    return job_ms, norm_ms, quant_ms, note


def roofline_of(gq, wk, job_ms, K, norm_ms, quant_ms, with_traffic):
    W, d, cfg = wk.W, wk.d, wk.cfg
    p1, p2 = algorithmic_bytes(gq, cfg, W, d)
    ms_per_step = job_ms / K
    q_avg = sum(quant_ms) / len(quant_ms)
    n_avg = sum(norm_ms) / len(norm_ms)
    peak, peak_kind = measured_hbm_peak()
    achieved = p2 / (q_avg * 1e-3) / 1e9
    traffic = recorded_traffic(wk.name, d) if with_traffic else None
    return {"bound": "hbm", "kernel": "fused pass of gq_quantize_aggregate "
                                      "(quant_tma_kernel when d % 4 == 0 and the rows fit)",
            "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "peak_source": f"{peak_kind} (hbm_gbs)",
            "traffic": None if traffic is None else round(traffic),
            "algorithmic_bytes": p2, "avg_launch_ms": round(q_avg, 5),
            "norm_kernel": {"achieved": round(p1 / (n_avg * 1e-3) / 1e9, 1),
                            "frac": round(p1 / (n_avg * 1e-3) / 1e9 / peak, 4),
                            "algorithmic_bytes": p1, "avg_launch_ms": round(n_avg, 5)},
            "step": {"achieved": round((p1 + p2) / (ms_per_step * 1e-3) / 1e9, 1),
                     "frac": round((p1 + p2) / (ms_per_step * 1e-3) / 1e9 / peak, 4),
                     "frac_of_8000": round((p1 + p2) / (ms_per_step * 1e-3) / 1e9 / 8000, 4)}}


def l2_flusher(dev):
    """Writes a buffer twice the size of L2, evicting whatever the last step left."""
    junk = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)

    def flush():
        junk.fill_(1.0)
    return flush


def run_ours(args, rank, world, local_rank):
    import allreduce_compatible_gradient_global_b200 as gq
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wk = Workload(gq, args.workload, dev, d=args.coords)
    W, d, cfg = wk.W, wk.d, wk.cfg
    K = args.steps
    grad_bytes = 4 * W * d
    flush = l2_flusher(dev) if grad_bytes < 2 * L2_BYTES else None
    sampler = ClockSampler(local_rank)
    sampler.start()
    job_ms, norm_ms, quant_ms, note = time_workload(wk, K, args.warmup, world, flush)
    # the fused pass without materialised codes (the sum-based exchange needs none)
    Knc = K if not wk.fresh else min(K, 5)
    n0, n1 = _events(2)
    _sync(world)
    n0.record(wk.stream)
    for i in range(Knc):
        wk.step(args.warmup + 2 * K + i, codes=False)
    n1.record(wk.stream)
    _sync(world)
    sampler.stop()
    nc_ms = job_time_ms(n0.elapsed_time(n1), world, dev)
    ms_per_step = job_ms / K
    value = job_gbs(grad_bytes, K, job_ms, world)
    roofline = roofline_of(gq, wk, job_ms, K, norm_ms, quant_ms, with_traffic=not args.coords)
    p1, p2 = algorithmic_bytes(gq, cfg, W, d)
    peak = roofline["peak"]
    p2_nc = p2 - W * gq.gq_packed_row_bytes(cfg, d)
    without_codes = {"value": round(job_gbs(grad_bytes, Knc, nc_ms, world), 2), "unit": "GB/s",
                     "ms_per_step": round(nc_ms / Knc, 5), "steps": Knc,
                     "algorithmic_bytes": p1 + p2_nc,
                     "step_frac": round((p1 + p2_nc) / (nc_ms / Knc * 1e-3) / 1e9 / peak, 4)}
    e2e = None if args.no_e2e else run_e2e(gq, args, wk, world, dev)
    data = {"normal_seg_d2^30_w8_ef": "synthetic (seeded per-2^20-segment sigma_k*N(0,1) "
                                      "gradients, a fresh draw every step)",
            "resnet50_t3_w8": "synthetic (seeded per-segment Student-t(3) gradients, "
                              "ResNet-50-sized)"}.get(args.workload, "synthetic")
    result = dict(
        metric=METRIC, value=round(value, 2), unit="GB/s", n_gpus=world, steps=K,
        warmup=args.warmup, ms_per_step=round(ms_per_step, 5), higher_is_better=True,
        scaling="weak", vs_baseline=None, dtype="f32", data=data,
        config={"workload": args.workload, "W": W, "d": d, "levels": cfg.levels, "s": cfg.s,
                "L": cfg.L, "bits": cfg.bits, "wire": cfg.wire, "scale": cfg.scale_kind,
                "ef": cfg.ef, "fresh_gradient_per_step": wk.fresh,
                "parallelism": f"replicas x{world}", "truncated_to_coords": args.coords,
                "l2": (f"inputs exceed L2: {grad_bytes / 1e6:.1f} MB of gradient per read vs "
                       f"{L2_BYTES / 1e6:.0f} MB L2") if flush is None else
                      "L2 flushed between timed steps (a 2x-L2 buffer written)"},
        roofline=roofline, gpu_launches=2 * K, clocks=sampler.summary(), e2e=e2e,
        timing=note, fused_without_codes=without_codes)
    wk.free()
    return result


def run_e2e(gq, args, wk, world, dev):
    """The same metric end to end: every step uploads its gradients from pinned
    host memory, runs both kernels and reads the decoded mean and the scale back
    into pinned host memory; host <-> device copies inside the timed region.

    Where a second gradient buffer fits the device, the steps are pipelined as a
    training loop would pipeline them: step i+1's upload (a copy stream, into the
    other gradient buffer) overlaps step i's kernels (gq_global_norm +
    gq_quantize_aggregate on the compute stream) and its read-back (a third
    stream).  The error rows, codes, sum and mean are the workload's one buffer
    set, so error feedback runs exactly as in consecutive steps; events order
    each buffer's writer after its last reader.  Otherwise gq_step_fused_host
    runs each step on one stream, the upload landing in the workload's own
    gradient buffer."""
    W, d, cfg, g, buf = wk.W, wk.d, wk.cfg, wk.g, wk.buf
    # every rank on this host pins its gradient and mean: refuse (and say why)
    # rather than exhaust the host's memory when the ranks together cannot
    need = (4 * W * d + 8 * d) * int(os.environ.get("LOCAL_WORLD_SIZE", world))
    fits, avail = host_buffers_fit(need, world, dev)
    if not fits:
        return {"value": None, "unit": "GB/s", "h2d_bytes_per_step": 4 * W * d,
                "d2h_bytes_per_step": 4 * d + 4,
                "skipped": f"pinned host buffers for the ranks on this host ({need / 2**30:.0f} "
                           f"GiB) exceed 80% of its available memory"
                           + ("" if avail is None else f" ({avail / 2**30:.0f} GiB on this rank)")}
    g_host = torch.empty((W, d), dtype=torch.float32, pin_memory=True)
    g_host.copy_(g)
    out_host = torch.empty(d, dtype=torch.float32, pin_memory=True)
    scale_host = torch.empty(1, dtype=torch.float32, pin_memory=True)
    free_b, _ = torch.cuda.mem_get_info(dev)
    pipelined = free_b > 4 * W * d + (2 << 30)
    K = max(1, min(args.steps, 8))
    if pipelined:
        gbufs = [g, torch.empty_like(g)]
        s_in, s_comp, s_out = torch.cuda.Stream(device=dev), wk.stream, torch.cuda.Stream(
            device=dev)
        nsteps = 2 + K
        h2d = [torch.cuda.Event() for _ in range(nsteps)]
        comp = [torch.cuda.Event() for _ in range(nsteps)]
        d2h = [torch.cuda.Event() for _ in range(nsteps)]

        def one(i):
            gb = gbufs[i % 2]
            if i >= 2:
                s_in.wait_event(comp[i - 2])  # step i-2's kernels were this buffer's readers
            with torch.cuda.stream(s_in):
                gb.copy_(g_host, non_blocking=True)
            h2d[i].record(s_in)
            s_comp.wait_event(h2d[i])
            if i >= 1:
                s_comp.wait_event(d2h[i - 1])  # the mean and scale have been read back
            cfg.step = 1000 + i
            gq.gq_global_norm(gb, buf.e if cfg.ef else None, cfg, buf.scale, buf.norms, buf.ws,
                              s_comp)
            gq.gq_quantize_aggregate(gb, buf.e, cfg, buf.scale, buf.codes, buf.sum, buf.out,
                                     buf.ws, s_comp)
            comp[i].record(s_comp)
            s_out.wait_event(comp[i])
            with torch.cuda.stream(s_out):
                out_host.copy_(buf.out, non_blocking=True)
                scale_host.copy_(buf.scale, non_blocking=True)
            d2h[i].record(s_out)

        for i in range(2):
            one(i)
        _sync(world)
        t0, t1 = _events(2)
        t0.record(s_in)
        for i in range(2, 2 + K):
            one(i)
        t1.record(s_out)
        torch.cuda.synchronize()
        api = ("pipelined: gradient upload on a copy stream into two alternating device "
               "buffers, gq_global_norm + gq_quantize_aggregate on the compute stream, mean "
               "and scale read back on a third stream")
        # the bound: the same upload alone, over the host link
        u0, u1 = _events(2)
        u0.record(s_in)
        with torch.cuda.stream(s_in):
            gbufs[1].copy_(g_host, non_blocking=True)
        u1.record(s_in)
        torch.cuda.synchronize()
        link_gbs = 4 * W * d / (u0.elapsed_time(u1) * 1e-3) / 1e9
    else:
        def one(i):
            cfg.step = 1000 + i
            gq.gq_step_fused_host(g_host, g, buf.e, cfg, buf.scale, buf.codes, buf.sum, buf.out,
                                  out_host, scale_host, buf.ws, wk.stream)

        one(0)
        _sync(world)
        t0, t1 = _events(2)
        t0.record(wk.stream)
        for i in range(1, 1 + K):
            one(i)
        t1.record(wk.stream)
        torch.cuda.synchronize()
        api = "gq_step_fused_host, one stream (a second gradient buffer does not fit)"
        link_gbs = None
    ms = job_time_ms(t0.elapsed_time(t1), world, dev)
    val = job_gbs(4 * W * d, K, ms, world)
    if gq.gq_get_device_status(buf.ws, wk.stream) != gq.GQ_OK:
        raise RuntimeError("device flag raised in the end-to-end run")
    del g_host
    out = {"value": round(val, 3), "unit": "GB/s", "h2d_bytes_per_step": 4 * W * d,
           "d2h_bytes_per_step": 4 * d + 4, "ms_per_step": round(ms / K, 4), "steps": K,
           "api": api}
    if link_gbs is not None:  # this rank's upload alone; the value is the whole job's
        out["host_link_upload_gbs"] = round(link_gbs, 2)
        out["frac_of_host_link"] = round(val / world / link_gbs, 4)
    return out


def host_buffers_fit(need, world, device):
    """Whether `need` bytes of pinned host buffers (every local rank's) fit in 80%
    of the host's available memory, decided once for all ranks: each measures
    after a barrier (before any rank pins) and the answer is the MIN over ranks,
    so every rank takes the same collective steps afterwards.  Returns
    (fits, this rank's available bytes or None)."""
    if world > 1:
        torch.distributed.barrier()
    avail = host_available_bytes()
    fits = avail is None or need <= 0.8 * avail
    if world > 1:
        flag = torch.tensor([1 if fits else 0], dtype=torch.int32, device=device)
        torch.distributed.all_reduce(flag, op=torch.distributed.ReduceOp.MIN)
        fits = bool(flag.item())
    return fits, avail


def host_available_bytes():
    """Available host memory (bytes), or None if it cannot be read."""
    try:
        import psutil
        return int(psutil.virtual_memory().available)
    except Exception:
        try:
            with open("/proc/meminfo") as f:
                for line in f:
                    if line.startswith("MemAvailable:"):
                        return int(line.split()[1]) * 1024
        except OSError:
            return None
    return None


def host_threads():
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else \
        (os.cpu_count() or 1)


_CPU_SAMPLE = {}


def cpu_sample(name, sample_coords):
    """The host sample of a workload (drawn once, shared by both CPU figures)."""
    wl = synthetic.WORKLOADS[name]
    W, d = wl["W"], wl["d"]
    n = d if sample_coords is None else min(d, sample_coords)
    key = (name, n)
    if key not in _CPU_SAMPLE:
        _CPU_SAMPLE.clear()
        g = synthetic.workload_gradients(name, device="cpu", d=n).numpy()
        e = np.zeros_like(g) if wl["ef"] else None
        _CPU_SAMPLE[key] = (g, e)
    g, e = _CPU_SAMPLE[key]
    return wl, W, d, n, g, e


def _sample_words(name, W, d, n, dt, extra=""):
    whole = n == d
    txt = (f"one oracle step (scale, codes, pack, sum, decode{', error feedback' if extra else ''})"
           f" on W={W} x {n} coordinates of the {name} recipe")
    if whole:
        return txt + f" (the full workload), {dt:.1f} s"
    return (txt + f" (a prefix; the per-coordinate cost does not depend on d, so the GB/s "
                  f"figure is extrapolated to the full d={d}), {dt:.1f} s")


def cpu_baseline(name, sample_coords=None):
    """The oracle as it stands (single-threaded C) on a sample of the workload."""
    import oracle
    wl, W, d, n, g, e = cpu_sample(name, sample_coords)
    kw = oracle_kwargs(wl)
    oracle.lib()
    t = time.perf_counter()
    oracle.step(g, e, ef=wl["ef"], **kw)
    dt = time.perf_counter() - t
    return {"value": round(4 * W * n / dt / 1e9, 4), "unit": "GB/s", "cores": 1,
            "kind": "oracle", "extrapolated": n != d,
            "sample": _sample_words(name, W, d, n, dt, "ef" if wl["ef"] else "")}


def oracle_step_threaded(g, threads, e=None, *, levels, s, L, scale_kind, bits, seed, step=0):
    """The oracle's step on `threads` host threads, for the threaded CPU figure.
    The oracle's scale is per worker (an fp64 sum in ascending coordinate order
    within a row, or the row's max |v|), so the rows run in parallel and S is
    the max of their scales.  With S fixed, every code depends only on its own
    coordinate (the uniforms are counter-based), so coordinate chunks of whole
    128-coordinate packing blocks are quantized at their own indices, packed,
    summed, decoded and (with e) error-fed independently.  The oracle's C
    routines release the GIL while they run.  Returns S, the packed rows, the
    integer sums, the mean and the new error rows (None without e)."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    W, d = g.shape
    per = -(-d // (threads * 4))
    step_c = max(128, -(-per // 128) * 128)
    bounds = [(c0, min(d, c0 + step_c)) for c0 in range(0, d, step_c)]

    def row_scale(w):
        return oracle.global_scale(g[w:w + 1], None if e is None else e[w:w + 1], scale_kind)[0]

    with ThreadPoolExecutor(max_workers=threads) as pool:
        S = np.float32(max(pool.map(row_scale, range(W))))

        def chunk(b):
            c0, c1 = b
            gs = g[:, c0:c1]
            es = None if e is None else e[:, c0:c1]
            codes = oracle.quantize(gs, es, levels=levels, s=s, L=L, seed=seed, step=step, S=S,
                                    js=np.arange(c0, c1, dtype=np.int64))
            packed = oracle.pack(codes, bits) if bits else None
            total = oracle.aggregate(codes, levels=levels, L=L)
            mean = oracle.decode_mean(total, W, levels=levels, s=s, L=L, S=S)
            e_new = None if e is None else oracle.error_feedback(gs, es, codes, levels=levels,
                                                                 s=s, L=L, S=S)
            return packed, total, mean, e_new

        parts = list(pool.map(chunk, bounds))
    packed = np.concatenate([x[0] for x in parts], axis=1) if bits else None
    e_new = None if e is None else np.concatenate([x[3] for x in parts], axis=1)
    return dict(S=S, packed=packed, sum=np.concatenate([x[1] for x in parts]),
                out=np.concatenate([x[2] for x in parts]), e=e_new)


def cpu_baseline_threads(name, sample_coords=None):
    """The same oracle step run coordinate-parallel over every host core the
    process may use (oracle_step_threaded): a second, fairer CPU figure."""
    import oracle
    wl, W, d, n, g, e = cpu_sample(name, sample_coords)
    kw = oracle_kwargs(wl)
    threads = host_threads()
    oracle.lib()
    t = time.perf_counter()
    oracle_step_threaded(g, threads, e, **kw)
    dt = time.perf_counter() - t
    return {"value": round(4 * W * n / dt / 1e9, 4), "unit": "GB/s", "cores": threads,
            "kind": f"oracle x{threads} threads", "extrapolated": n != d,
            "sample": _sample_words(name, W, d, n, dt, "ef" if wl["ef"] else "")
            + f"; rows then coordinate chunks over {threads} threads"}


# ------------------------------------------------------- the other configurations
def measure_config(gq, name, K, warmup, dev, with_cpu):
    """value, roofline and CPU oracle of one fixed-gradient workload (one GPU)."""
    wk = Workload(gq, name, dev)
    flush = l2_flusher(dev) if 4 * wk.W * wk.d < 2 * L2_BYTES else None
    job_ms, norm_ms, quant_ms, note = time_workload(wk, K, warmup, 1, flush)
    roof = roofline_of(gq, wk, job_ms, K, norm_ms, quant_ms, with_traffic=True)
    cfg = wk.cfg
    res = {"value": round(job_gbs(4 * wk.W * wk.d, K, job_ms, 1), 2), "unit": "GB/s",
           "ms_per_step": round(job_ms / K, 5), "steps": K, "W": wk.W, "d": wk.d,
           "levels": cfg.levels, "s": cfg.s, "L": cfg.L, "bits": cfg.bits, "wire": cfg.wire,
           "scale": cfg.scale_kind, "ef": cfg.ef, "roofline": roof, "timing": note,
           "gpu_launches": 2 * K}
    wk.free()
    if with_cpu:
        res["cpu_baseline"] = cpu_baseline(name, CPU_SAMPLE_COORDS.get(name))
    return res


def recorded_logq_counts(rank):
    """Thread instructions per launch of the two log-quantizer kernels at this
    rank (ncu, committed), if taken on the current sources; else None."""
    try:
        with open(LOGQ_COUNTS_FILE) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    if rec.get("source_hash") != source_hash(LOGQ_SOURCES):
        return None
    return rec.get("ranks", {}).get(str(rank))


def issue_peak_ginst():
    """G thread instructions per second the SMs can issue at their maximum clock."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            mhz = float(json.load(f)["sm_max_mhz"])
    except (OSError, KeyError, ValueError):
        mhz = 1965.0
    sms = torch.cuda.get_device_properties(0).multi_processor_count \
        if torch.cuda.is_available() else SM_COUNT_B200
    return sms * ISSUE_PER_SM_PER_CLK * mhz * 1e-3


def lq_bytes(W, n, nmats):
    """Algorithmic bytes of the log quantizer on W workers x n factor entries
    (nmats matrices per worker): the quantize pass reads the factors once and
    writes int8 codes and the per-matrix max; the decode-sum reads the codes
    and the max and writes the fp32 sum."""
    q = 4 * W * n + W * n + 4 * W * nmats
    dsum = W * n + 4 * W * nmats + 4 * n
    return q, dsum


def measure_lq(gq, r, K, dev, with_cpu):
    """The log quantizer on W = 8 workers x 24 factor pairs of 4096 x r:
    quantize + decode-sum per step, each timed by events, L2 flushed between
    steps (the factors fit in L2)."""
    W = synthetic.LQ_WORKLOAD["W"]
    alpha = synthetic.LQ_WORKLOAD["alpha"]
    x, sizes = synthetic.lq_factors(r, W=W, device=dev)
    n = x.shape[1]
    nm = len(sizes)
    R = [4096] * nm
    C = [r] * nm
    cfg = gq.GQConfig(levels="log", alpha=alpha, seed=1)
    mx = torch.empty((W, nm), dtype=torch.float32, device=dev)
    codes = torch.empty((W, n), dtype=torch.int8, device=dev)
    out = torch.empty(n, dtype=torch.float32, device=dev)
    ws = torch.empty(gq.gq_workspace_bytes(gq.GQConfig(), W, 1), dtype=torch.uint8, device=dev)
    gq.gq_workspace_init(ws)
    flush = l2_flusher(dev)
    st = torch.cuda.current_stream()
    evs = [_events(3) for _ in range(K + 3)]
    for i in range(K + 3):
        flush()
        cfg.step = i
        evs[i][0].record(st)
        gq.gq_logq_quantize(x, R, C, cfg, mx, codes, ws, st)
        evs[i][1].record(st)
        gq.gq_logq_decode_sum(codes, mx, R, C, cfg, out, st)
        evs[i][2].record(st)
    torch.cuda.synchronize()
    if gq.gq_get_device_status(ws, st) != gq.GQ_OK:
        raise RuntimeError("device flag raised in the log-quantizer run")
    qm = sum(e[0].elapsed_time(e[1]) for e in evs[3:]) / K
    dm = sum(e[1].elapsed_time(e[2]) for e in evs[3:]) / K
    step_ms = qm + dm
    qb, db = lq_bytes(W, n, nm)
    peak, peak_kind = measured_hbm_peak()
    # The quantize kernel is bound by instruction issue (a log1p, two divisions
    # and a quarter of a Philox call per entry), not by HBM: its roofline is
    # thread instructions executed (ncu, committed) per second against the
    # issue peak; the HBM figures stand beside it.
    counts = recorded_logq_counts(r)
    ipeak = issue_peak_ginst()
    hbm = {"achieved": round(qb / (qm * 1e-3) / 1e9, 1), "peak": peak, "unit": "GB/s",
           "frac": round(qb / (qm * 1e-3) / 1e9 / peak, 4),
           "peak_source": f"{peak_kind} (hbm_gbs)", "algorithmic_bytes": qb}
    if counts is not None:
        qi = float(counts["quantize_thread_inst"])
        roof = {"bound": "alu", "kernel": "logq_quantize_kernel",
                "achieved": round(qi / (qm * 1e-3) / 1e9, 1), "peak": round(ipeak, 1),
                "unit": "G thread-instr/s", "frac": round(qi / (qm * 1e-3) / 1e9 / ipeak, 4),
                "peak_source": "derived: SMs x 4 schedulers x 32 lanes x max SM clock",
                "instructions": int(qi), "instructions_per_entry": round(qi / (W * n), 2),
                "traffic": counts.get("quantize_dram_bytes"), "hbm": hbm}
    else:
        roof = dict(hbm, bound="hbm", kernel="logq_quantize_kernel", traffic=None,
                    note="no instruction count recorded for the current log-quantizer source")
    roof.update({"avg_launch_ms": round(qm, 5),
                 "decode_sum_kernel": {
                     "achieved": round(db / (dm * 1e-3) / 1e9, 1),
                     "frac": round(db / (dm * 1e-3) / 1e9 / peak, 4),
                     "algorithmic_bytes": db, "avg_launch_ms": round(dm, 5)},
                 "step_hbm": {"achieved": round((qb + db) / (step_ms * 1e-3) / 1e9, 1),
                              "frac": round((qb + db) / (step_ms * 1e-3) / 1e9 / peak, 4)}})
    res = {"value": round(4 * W * n / (step_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
           "ms_per_step": round(step_ms, 5), "steps": K, "rank": r, "W": W,
           "elements_per_worker": n, "matrices_per_worker": nm, "roofline": roof,
           "timing": "each step's two kernels timed by CUDA events; L2 flushed between steps",
           "code_bytes_per_worker": n, "fp32_bytes_per_worker": 4 * n}
    if with_cpu:
        res["cpu_baseline"] = cpu_baseline_lq(x.cpu().numpy(), sizes, alpha)
    del x, mx, codes, out, ws
    torch.cuda.empty_cache()
    return res


def cpu_baseline_lq(x, sizes, alpha):
    import oracle
    W, n = x.shape
    oracle.lib()
    t = time.perf_counter()
    mx, codes = oracle.logq_quantize(x, sizes, alpha=alpha, seed=1, step=0)
    oracle.logq_decode_sum(codes, mx, sizes, alpha=alpha)
    dt = time.perf_counter() - t
    return {"value": round(4 * W * n / dt / 1e9, 4), "unit": "GB/s", "cores": 1,
            "kind": "oracle", "extrapolated": False,
            "sample": f"one oracle log-quantize + decode-sum of all W={W} x {n} factor "
                      f"entries (the full workload), {dt:.2f} s"}


def run_extras(args, dev):
    import allreduce_compatible_gradient_global_b200 as gq
    K = max(10, min(args.steps, 50))
    out = {}
    for name in EXTRA_WORKLOADS:
        out[name] = measure_config(gq, name, K, args.warmup, dev, not args.no_cpu_baseline)
    for r in synthetic.LQ_WORKLOAD["ranks"]:
        out[f"lq_r{r}_w8"] = measure_lq(gq, r, K, dev, not args.no_cpu_baseline)
    return out


# --------------------------------------------------------------- reference arm
def run_reference(args):
    """Reference arm: the CPU oracle, each step a bounded sample of the
    workload (a prefix of reference_coords coordinates, a fresh draw every step
    when the workload has one, error buffers carried over)."""
    import oracle
    wl = synthetic.WORKLOADS[args.workload]
    W, d = wl["W"], wl["d"]
    n = min(d, args.reference_coords)
    fresh = bool(wl.get("fresh_per_step", False))
    kw = oracle_kwargs(wl)
    g = synthetic.workload_gradients(args.workload, device="cpu", d=n).numpy()
    e = np.zeros_like(g) if wl["ef"] else None
    oracle.lib()
    dt = 0.0
    for i in range(args.warmup + args.steps):
        if fresh and i > 0:
            g = synthetic.workload_gradients(args.workload, device="cpu", d=n, step=i).numpy()
        t = time.perf_counter()
        res = oracle.step(g, e, step=i, ef=wl["ef"], **kw)
        if i >= args.warmup:
            dt += time.perf_counter() - t
        if wl["ef"]:
            e = res["e"]
    value = 4 * W * n * args.steps / dt / 1e9
    sample = (f"each step: one oracle step on W={W} x {n} coordinates (a prefix of the "
              f"{args.workload} recipe, d={d}"
              + (", a fresh draw every step, error buffers carried over" if fresh else "")
              + "; the prefix's draw is untimed)")
    return dict(metric=METRIC, value=round(value, 4), unit="GB/s", n_gpus=args.gpus,
                steps=args.steps, warmup=args.warmup, ms_per_step=round(dt / args.steps * 1e3, 3),
                higher_is_better=True, scaling="weak", vs_baseline=None, dtype="f32",
                data="synthetic", impl="reference",
                config={"workload": args.workload, "W": W, "d": d, "sample_coords": n},
                cpu_baseline={"value": round(value, 4), "unit": "GB/s", "cores": 1,
                              "kind": "oracle", "sample": sample},
                e2e={"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                     "d2h_bytes_per_step": 0})


# ------------------------------------------------------------------ other modes
SWEEP_ORACLE_COORDS = 1 << 20


def sweep_oracle(g, ef):
    """The oracle's step on a prefix of a sweep row's gradient (CPU, one thread)."""
    import oracle
    W, d = g.shape
    n = min(d, SWEEP_ORACLE_COORDS)
    gh = g[:, :n].cpu().numpy()
    eh = np.zeros_like(gh) if ef else None
    oracle.lib()
    t = time.perf_counter()
    oracle.step(gh, eh, levels=0, s=15, scale_kind=0, seed=0x5EED, ef=ef, bits=5)
    dt = time.perf_counter() - t
    return {"value": round(4 * W * n / dt / 1e9, 4), "unit": "GB/s", "coords": n}


def time_step_pair(gq, g, e, cfg, buf, K, warmup, stream):
    """Median per-kernel times and the mean step time (ms) of norm + fused pass.
    The step time comes from K steps with events around the run only; the
    per-kernel medians from K further steps with an event around each kernel."""
    def step(i, ev=None):
        cfg.step = i
        if ev is not None:
            ev[0].record(stream)
        gq.gq_global_norm(g, e if cfg.ef else None, cfg, buf.scale, buf.norms, buf.ws, stream)
        if ev is not None:
            ev[1].record(stream)
        gq.gq_quantize_aggregate(g, e, cfg, buf.scale, buf.codes, buf.sum, buf.out, buf.ws, stream)
        if ev is not None:
            ev[2].record(stream)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(K):
        step(warmup + i)
    t1.record(stream)
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    for i in range(K):
        step(warmup + K + i, evs[i])
    torch.cuda.synchronize()
    if gq.gq_get_device_status(buf.ws, stream) != gq.GQ_OK:
        raise RuntimeError("device flag raised during the sweep")
    n = statistics.median(e[0].elapsed_time(e[1]) for e in evs)
    q = statistics.median(e[1].elapsed_time(e[2]) for e in evs)
    return n, q, t0.elapsed_time(t1) / K


def time_step_graph(gq, g, cfg, W, d, K):
    """Mean step time (ms) of the step captured once in a CUDA graph (norm pass,
    fused pass, device step counter advanced in the graph) and replayed K times."""
    step_dev = torch.zeros(1, dtype=torch.int32, device=g.device)
    gcfg = gq.GQConfig(levels=cfg.levels, s=cfg.s, L=cfg.L, bits=cfg.bits,
                       scale_kind=cfg.scale_kind, wire=cfg.wire, ef=cfg.ef, seed=cfg.seed,
                       step_dev=step_dev)
    buf = gq.StepBuffers(gcfg, W, d)
    gq.gq_step_fused(g, buf.e, gcfg, buf.scale, buf.norms, buf.codes, buf.sum, buf.out, buf.ws)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        gq.gq_step_fused(g, buf.e, gcfg, buf.scale, buf.norms, buf.codes, buf.sum, buf.out,
                         buf.ws)
        gq.gq_advance_step(step_dev)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(K):
        graph.replay()
    t1.record()
    torch.cuda.synchronize()
    if gq.gq_get_device_status(buf.ws) != gq.GQ_OK:
        raise RuntimeError("device flag raised in the graph replay")
    ms = t0.elapsed_time(t1) / K
    del graph, buf
    return ms


def run_sweep(args):
    """Step throughput over d = 2^16 ... 2^30 at W = 8 (uniform s = 15, 5-bit
    codes, int8 sums, L2 scale), error feedback off and on.  Below ~2^22 the
    second read can hit L2; the fraction is reported but not targeted there.
    Each row also times the step captured in a CUDA graph and replayed, which
    removes the host's per-call cost where the step is launch-bound."""
    import allreduce_compatible_gradient_global_b200 as gq
    torch.cuda.set_device(0)
    stream = torch.cuda.current_stream()
    peak, peak_kind = measured_hbm_peak()
    rows = []
    W = 8
    sampler = ClockSampler(0)   # sm_mhz of a row: median clock over its timed steps
    sampler.start()
    for ef in (False, True):
        for lg in range(16, 31, 2):
            d = 1 << lg
            cfg = gq.GQConfig(levels="uniform", s=15, bits=5, wire="int8", scale_kind="l2", ef=ef,
                              seed=0x5EED)
            g = synthetic.make_gradients(W, d, "normal", seed=lg, device="cuda")
            buf = gq.StepBuffers(cfg, W, d)
            K = max(20, min(400, int(2e9 // (4 * W * d))))
            sampler.samples.clear()
            sampler.times.clear()
            t_row = time.perf_counter()
            n_ms, q_ms, step_ms = time_step_pair(gq, g, buf.e, cfg, buf, K, 5, stream)
            row_mhz = sampler.median_between(t_row, time.perf_counter())
            graph_ms = time_step_graph(gq, g, cfg, W, d, K)
            p1, p2 = algorithmic_bytes(gq, cfg, W, d)
            ora = None if args.no_cpu_baseline else sweep_oracle(g, ef)
            rows.append({"d": d, "log2_d": lg, "ef": ef, "steps": K, "oracle": ora,
                         "step_ms": round(step_ms, 5), "norm_ms": round(n_ms, 5),
                         "quant_ms": round(q_ms, 5),
                         "grad_gbs": round(4 * W * d / (step_ms * 1e-3) / 1e9, 1),
                         "step_frac": round((p1 + p2) / (step_ms * 1e-3) / 1e9 / peak, 4),
                         "quant_frac": round(p2 / (q_ms * 1e-3) / 1e9 / peak, 4),
                         "graph_step_ms": round(graph_ms, 5),
                         "graph_grad_gbs": round(4 * W * d / (graph_ms * 1e-3) / 1e9, 1),
                         "sm_mhz": row_mhz})
            del g, buf
            torch.cuda.empty_cache()
    sampler.stop()
    return {"metric": METRIC, "mode": "sweep", "unit": "GB/s", "peak": peak,
            "peak_source": peak_kind, "W": W, "config": "uniform s=15, 5-bit, int8 sum, L2",
            "oracle": None if args.no_cpu_baseline else
            {"kind": "oracle", "cores": 1,
             "sample": f"each row: one oracle step on a prefix of min(d, {SWEEP_ORACLE_COORDS}) "
                       "coordinates of the row's gradient (all 8 workers), single-threaded; "
                       "GB/s of fp32 gradient"},
            "sweep": rows}


def time_launch_series(gq, sampler, d, n, idle_s):
    """n fused passes (W = 8, uniform s = 15, 5-bit codes, int8 sums, L2 scale,
    no error feedback) launched back to back after idle_s seconds of idle GPU:
    per launch its fraction of the copy figure and the median SM clock while it
    ran (the launch's device interval placed on the host clock from the series'
    first event)."""
    W = 8
    cfg = gq.GQConfig(levels="uniform", s=15, bits=5, wire="int8", scale_kind="l2", seed=0x5EED)
    g = synthetic.make_gradients(W, d, "normal", seed=3, device="cuda")
    buf = gq.StepBuffers(cfg, W, d)
    gq.gq_global_norm(g, None, cfg, buf.scale, buf.norms, buf.ws)
    for i in range(3):
        gq.gq_quantize_aggregate(g, None, cfg, buf.scale, buf.codes, buf.sum, buf.out, buf.ws)
    torch.cuda.synchronize()
    time.sleep(idle_s)
    ev = _events(n + 1)
    stream = torch.cuda.current_stream()
    t0 = time.perf_counter()
    ev[0].record(stream)
    for i in range(n):
        cfg.step = 3 + i
        gq.gq_quantize_aggregate(g, None, cfg, buf.scale, buf.codes, buf.sum, buf.out, buf.ws)
        ev[i + 1].record(stream)
    torch.cuda.synchronize()
    if gq.gq_get_device_status(buf.ws) != gq.GQ_OK:
        raise RuntimeError("device flag raised in the launch series")
    _, p2 = algorithmic_bytes(gq, cfg, W, d)
    peak, _ = measured_hbm_peak()
    launches = []
    for i in range(n):
        a = ev[0].elapsed_time(ev[i]) * 1e-3
        ms = ev[i].elapsed_time(ev[i + 1])
        launches.append((p2 / (ms * 1e-3) / 1e9 / peak,
                         sampler.median_between(t0 + a, t0 + a + ms * 1e-3)))
    del g, buf
    torch.cuda.empty_cache()
    return launches


def run_power(args):
    """The fused pass without error feedback is bound by instruction issue, so
    its speed follows the SM clock, which the 1 kW power cap lowers under
    sustained load.  The same launch at d = 2^26 is timed as a short burst and
    as a sustained series, and at d = 2^30 as a series: per segment the median
    fraction of the copy figure and the median SM clock, and the fraction
    scaled to the maximum clock."""
    import allreduce_compatible_gradient_global_b200 as gq
    torch.cuda.set_device(0)
    sampler = ClockSampler(0)
    sampler.start()
    series = [(1 << 26, 20), (1 << 26, 600), (1 << 30, 40)]
    rows = []
    try:
        for d, n in series:
            launches = time_launch_series(gq, sampler, d, n, 1.0)
            for name, part in (("first 5", launches[:5]), ("first 20", launches[:20]),
                               ("last 20", launches[-20:])):
                fr = statistics.median(f for f, _ in part)
                mhz = [m for _, m in part if m is not None]
                mhz = statistics.median(mhz) if mhz else None
                rows.append({"d": d, "launches": n, "segment": name, "frac": round(fr, 4),
                             "sm_mhz": mhz,
                             "frac_at_max_clock": (round(fr * sampler.max_mhz / mhz, 4)
                                                   if mhz and sampler.max_mhz else None)})
    finally:
        sampler.stop()
    return {"metric": "fused pass fraction of the measured copy figure against the SM clock",
            "mode": "power", "unit": "fraction", "config": "W=8, uniform s=15, 5-bit codes, "
            "int8 sums, L2 scale, no error feedback; 1 s idle before each series",
            "clocks": sampler.summary(), "rows": rows}


def run_buckets(args):
    """Per-bucket scales on the benchmark workload: the global-scale step against
    steps with one scale per bucket of 2^b coordinates.  Per variant: median
    per-launch times of the scale pass (both bucket launches together) and of
    the fused pass, the step's gradient GB/s, and the relative squared error
    ||out - mean_w g||^2 / ||mean_w g||^2 of the decoded mean (one draw),
    which is what the finer scales buy."""
    import allreduce_compatible_gradient_global_b200 as gq
    torch.cuda.set_device(0)
    stream = torch.cuda.current_stream()
    peak, peak_kind = measured_hbm_peak()
    wl, cfg = workload_config(gq, args.workload)
    W, d = wl["W"], wl["d"]
    g = synthetic.workload_gradients(args.workload, device="cuda")
    e = torch.zeros_like(g) if cfg.ef else None
    gbar = g.double().mean(dim=0)
    ref2 = float((gbar * gbar).sum())
    p1, p2 = algorithmic_bytes(gq, cfg, W, d)
    K = max(20, min(args.steps, 200))
    rows = []
    for b in (None, 10, 12, 14, 17, 20):
        if b is None:
            buf = gq.StepBuffers(cfg, W, d)
            ws = buf.ws
            table = None
        else:
            buf = gq.StepBuffers(cfg, W, d)
            nk = gq.gq_bucket_count(d, b)
            table = torch.empty(3 * nk, dtype=torch.float32, device="cuda")
            ws = torch.empty(gq.gq_bucket_workspace_bytes(cfg, W, d, b), dtype=torch.uint8,
                             device="cuda")
            gq.gq_workspace_init(ws)

        def one(i, ev=None):
            cfg.step = i
            if ev is not None:
                ev[0].record(stream)
            if b is None:
                gq.gq_global_norm(g, e, cfg, buf.scale, buf.norms, ws, stream)
            else:
                gq.gq_bucket_scales(g, e, b, cfg, table, ws, stream)
            if ev is not None:
                ev[1].record(stream)
            if b is None:
                gq.gq_quantize_aggregate(g, e, cfg, buf.scale, buf.codes, buf.sum, buf.out, ws,
                                         stream)
            else:
                gq.gq_quantize_aggregate_bucketed(g, e, b, cfg, table, buf.codes, buf.sum,
                                                  buf.out, ws, stream)
            if ev is not None:
                ev[2].record(stream)

        for i in range(5):
            one(i)
        torch.cuda.synchronize()
        if e is not None:
            e.zero_()
        one(5)
        torch.cuda.synchronize()
        diff = buf.out.double() - gbar
        rel = float((diff * diff).sum()) / ref2
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
        for i in range(K):
            one(6 + i, evs[i])
        torch.cuda.synchronize()
        if gq.gq_get_device_status(ws, stream) != gq.GQ_OK:
            raise RuntimeError("device flag raised in the bucket comparison")
        sm = statistics.median(x[0].elapsed_time(x[1]) for x in evs)
        qm = statistics.median(x[1].elapsed_time(x[2]) for x in evs)
        step_ms = sum(x[0].elapsed_time(x[2]) for x in evs) / K
        rows.append({"bucket_log2": b, "buckets": 1 if b is None else gq.gq_bucket_count(d, b),
                     "scale_ms": round(sm, 5), "quant_ms": round(qm, 5),
                     "step_ms": round(step_ms, 5),
                     "grad_gbs": round(4 * W * d / (step_ms * 1e-3) / 1e9, 1),
                     "scale_frac": round(p1 / (sm * 1e-3) / 1e9 / peak, 4),
                     "quant_frac": round(p2 / (qm * 1e-3) / 1e9 / peak, 4),
                     "rel_sq_error": rel})
        del buf, table, ws
        torch.cuda.empty_cache()
    return {"metric": METRIC, "mode": "buckets", "unit": "GB/s", "peak": peak,
            "peak_source": peak_kind, "workload": args.workload, "W": W, "d": d, "rows": rows}


def run_lqsgd(args):
    """The whole LQ-SGD step (PowerSGD low rank + log quantizer on both
    factors, error feedback) on W = 8 workers x 24 matrices of 4096 x 4096,
    ranks 1, 4, 7: step time through gq_lqsgd_step, and the two passes over
    the matrices (gq_psgd_project, gq_psgd_back_project) timed alone against
    their algorithmic bytes."""
    import allreduce_compatible_gradient_global_b200 as gq
    torch.cuda.set_device(0)
    stream = torch.cuda.current_stream()
    peak, peak_kind = measured_hbm_peak()
    wl = synthetic.LQ_WORKLOAD
    W, L, n, m = wl["W"], args.lqsgd_mats, wl["n"], wl["m"]
    K = max(5, min(args.steps, 20))
    rows_out = []
    g = None
    ranks = wl["ranks"] if args.lqsgd_rank is None else (args.lqsgd_rank,)
    for r in ranks:
        sh = gq.PsgdShapes([n] * L, [m] * L, r)
        if g is None:
            g = synthetic.make_gradients(W, sh.total, "normal", seed=synthetic.seed_for(5),
                                         device="cuda")
            mst = torch.zeros_like(g)
        else:
            mst.zero_()
        p = torch.zeros(sh.ptotal, dtype=torch.float32, device="cuda")
        q = synthetic.make_gradients(1, sh.qtotal, "normal", seed=r, device="cuda")[0]
        ghat = torch.empty(sh.total, dtype=torch.float32, device="cuda")
        pw = torch.empty((W, sh.ptotal), dtype=torch.float32, device="cuda")
        qw = torch.empty((W, sh.qtotal), dtype=torch.float32, device="cuda")
        ws = torch.empty(gq.gq_psgd_workspace_bytes(W, sh), dtype=torch.uint8, device="cuda")
        gq.gq_workspace_init(ws)
        cfg = gq.GQConfig(levels="log", alpha=wl["alpha"], seed=1)
        for i in range(3):
            cfg.step = i
            gq.gq_lqsgd_step(g, mst, sh, i > 0, cfg, p, q, ghat, ws, stream)
        torch.cuda.synchronize()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        ev[0].record(stream)
        for i in range(K):
            cfg.step = 3 + i
            gq.gq_lqsgd_step(g, mst, sh, True, cfg, p, q, ghat, ws, stream)
        ev[1].record(stream)
        torch.cuda.synchronize()
        if gq.gq_get_device_status(ws, stream) != gq.GQ_OK:
            raise RuntimeError("device flag raised in the LQ-SGD step")
        step_ms = ev[0].elapsed_time(ev[1]) / K
        pj, bk = [], []
        for i in range(K):
            e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            e[0].record(stream)
            gq.gq_psgd_project(g, mst, sh, True, p, q, pw, stream)
            e[1].record(stream)
            gq.gq_psgd_back_project(mst, p, sh, qw, ws, stream)
            e[2].record(stream)
            pj.append(e)
        torch.cuda.synchronize()
        proj_ms = statistics.median(e[0].elapsed_time(e[1]) for e in pj)
        back_ms = statistics.median(e[1].elapsed_time(e[2]) for e in pj)
        wt = W * sh.total
        proj_bytes = 12 * wt + 4 * W * sh.ptotal
        back_bytes = 4 * wt
        step_bytes = 16 * wt + 4 * sh.total
        rows_out.append({
            "rank": r, "step_ms": round(step_ms, 4),
            "grad_gbs": round(4 * wt / (step_ms * 1e-3) / 1e9, 1),
            "step_frac": round(step_bytes / (step_ms * 1e-3) / 1e9 / peak, 4),
            "project_ms": round(proj_ms, 4),
            "project_frac": round(proj_bytes / (proj_ms * 1e-3) / 1e9 / peak, 4),
            "back_project_ms": round(back_ms, 4),
            "back_project_frac": round(back_bytes / (back_ms * 1e-3) / 1e9 / peak, 4),
            "wire_bytes_per_worker": (sh.ptotal + sh.qtotal),
            "fp32_bytes_per_worker": 4 * sh.total})
        del p, q, ghat, pw, qw, ws
    del g, mst
    torch.cuda.empty_cache()
    return {"metric": "LQ-SGD step: fp32 gradient GB/s", "mode": "lqsgd", "unit": "GB/s",
            "peak": peak, "peak_source": peak_kind, "W": W,
            "matrices": f"{L} x {n}x{m} per worker", "rows": rows_out}


def run_dp(args, rank, world, local_rank):
    """The real data-parallel exchange (one worker per rank, NCCL): per step
    gq_global_norm + MAX all-reduce of the scale + gq_quantize_aggregate + SUM
    all-reduce of the int8 sums + decode, against a plain fp32 SUM all-reduce of
    the same gradient.  Times are the max over ranks of CUDA-event times."""
    import allreduce_compatible_gradient_global_b200 as gq
    from allreduce_compatible_gradient_global_b200.dp import DataParallelStep
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream()
    wl, cfg = workload_config(gq, args.workload)
    d = args.coords or wl["d"]
    g = synthetic.make_gradients(1, d, wl["recipe"], seed=synthetic.seed_for(wl["seed_index"])
                                 + rank, device=dev, seg=wl.get("seg", 0), lo=wl.get("lo", 0.0),
                                 hi=wl.get("hi", 0.0))
    stepper = DataParallelStep(cfg, d, w_local=1, device=dev)
    chunked = DataParallelStep(cfg, d, w_local=1, device=dev, chunks=args.dp_chunks) \
        if args.dp_chunks > 1 else None
    flat = g[0].clone()
    K = args.steps

    def timed(fn):
        for i in range(args.warmup):
            fn(i)
        torch.distributed.barrier()
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for i in range(K):
            fn(args.warmup + i)
        t1.record(stream)
        torch.cuda.synchronize()
        return job_time_ms(t0.elapsed_time(t1), world, dev) / K

    q_ms = timed(lambda i: stepper(g, None, step=i))
    c_ms = timed(lambda i: chunked(g, None, step=i)) if chunked is not None else None
    f_ms = timed(lambda i: torch.distributed.all_reduce(flat))
    # the same exchanges captured once in a CUDA graph and replayed: one host
    # call per step, so the chunk loop no longer costs host time per chunk
    stepper.capture(g, None)
    qg_ms = timed(lambda i: stepper.replay())
    stepper.close()
    cg_ms = None
    if chunked is not None:
        chunked.capture(g, None)
        cg_ms = timed(lambda i: chunked.replay())
        chunked.close()
    best = min(x for x in (q_ms, c_ms, qg_ms, cg_ms) if x is not None)
    return {"metric": "data-parallel exchange: compressed step vs fp32 all-reduce",
            "mode": "dp", "n_gpus": world, "workload": args.workload, "d": d,
            "wire": "int8 sums via NCCL", "compressed_step_ms": round(q_ms, 5),
            "compressed_chunked_step_ms": None if c_ms is None else round(c_ms, 5),
            "compressed_graph_step_ms": round(qg_ms, 5),
            "compressed_chunked_graph_step_ms": None if cg_ms is None else round(cg_ms, 5),
            "chunks": args.dp_chunks, "fp32_allreduce_ms": round(f_ms, 5),
            "speedup": round(f_ms / best, 3),
            "bytes_on_wire_per_rank": {"compressed": d + 4, "fp32": 4 * d}}


def run_nat(args):
    """Natural compression on the bench workload (W = 8 x 25,557,032): per step
    gq_nat_quantize of every worker's row and gq_nat_decode_sum of the codes
    over workers (the gather-style exchange done on one GPU).  value and
    ms_per_step from K steps with events around the run only; per-kernel
    launch times from K further steps with events around each kernel."""
    import allreduce_compatible_gradient_global_b200 as gq
    torch.cuda.set_device(0)
    stream = torch.cuda.current_stream()
    wl = synthetic.WORKLOADS[args.workload]
    W, d = wl["W"], (args.coords or wl["d"])
    x = synthetic.workload_gradients(args.workload, device="cuda", d=d)
    codes = torch.empty((W, d), dtype=torch.int16, device="cuda")
    out = torch.empty(d, dtype=torch.float32, device="cuda")
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    gq.gq_workspace_init(ws)
    cfg = gq.GQConfig(levels="nat", seed=0x5EED)
    K = args.steps

    def step(i, ev=None):
        cfg.step = i
        if ev is not None:
            ev[0].record(stream)
        gq.gq_nat_quantize(x, cfg, codes, ws, stream)
        if ev is not None:
            ev[1].record(stream)
        gq.gq_nat_decode_sum(codes, out, stream)
        if ev is not None:
            ev[2].record(stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    sampler = ClockSampler(0)
    sampler.start()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(K):
        step(args.warmup + i)
    t1.record(stream)
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    for i in range(K):
        step(args.warmup + K + i, evs[i])
    torch.cuda.synchronize()
    sampler.stop()
    if gq.gq_get_device_status(ws, stream) != gq.GQ_OK:
        raise RuntimeError("non-finite input in the natural-compression run")
    ms = t0.elapsed_time(t1) / K
    q_ms = sum(e[0].elapsed_time(e[1]) for e in evs) / K
    s_ms = sum(e[1].elapsed_time(e[2]) for e in evs) / K
    peak, peak_kind = measured_hbm_peak()
    qb = 4 * W * d + 2 * W * d      # read x, write int16 codes
    sb = 2 * W * d + 4 * d          # read the codes, write the fp32 sum
    return {"metric": "natural compression: quantize + decode-sum, fp32 gradient GB/s",
            "mode": "nat", "unit": "GB/s", "workload": args.workload, "W": W, "d": d,
            "value": round(4 * W * d * 1e-9 / (ms * 1e-3), 2), "ms_per_step": round(ms, 5),
            "steps": K, "warmup": args.warmup,
            "quantize": {"avg_launch_ms": round(q_ms, 5), "algorithmic_bytes": qb,
                         "achieved_gbs": round(qb / (q_ms * 1e-3) / 1e9, 1),
                         "frac": round(qb / (q_ms * 1e-3) / 1e9 / peak, 4)},
            "decode_sum": {"avg_launch_ms": round(s_ms, 5), "algorithmic_bytes": sb,
                           "achieved_gbs": round(sb / (s_ms * 1e-3) / 1e9, 1),
                           "frac": round(sb / (s_ms * 1e-3) / 1e9 / peak, 4)},
            "peak": peak, "peak_source": f"{peak_kind} (hbm_gbs)",
            "wire_bytes_per_worker_coordinate": 2, "clocks": sampler.summary()}


def run_lq(args):
    """The LQ-SGD log quantizer: quantize + decode-sum of 24 factor pairs of
    4096 x r per worker, W = 8, r in {1, 4, 7}, with the roofline of both
    kernels and the oracle on the same factors."""
    import allreduce_compatible_gradient_global_b200 as gq
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    rows = [measure_lq(gq, r, max(10, args.steps), dev, not args.no_cpu_baseline)
            for r in synthetic.LQ_WORKLOAD["ranks"]]
    return {"metric": "LQ-SGD log quantizer: fp32 factor GB/s", "mode": "lq", "unit": "GB/s",
            "W": synthetic.LQ_WORKLOAD["W"], "rows": rows}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=None, choices=sorted(synthetic.WORKLOADS),
                    help=f"default: {DEFAULT_WORKLOAD} for the bench line and the reference "
                         f"arm, {MODE_WORKLOAD} for --buckets, --nat and --dp")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the other configurations (the \"configs\" key of the line)")
    ap.add_argument("--reference-coords", type=int, default=1 << 21)
    ap.add_argument("--coords", type=int, default=None,
                    help="truncate the workload to this many coordinates (a smaller case "
                         "of the same recipe, for profiling; not a bench line)")
    ap.add_argument("--sweep", action="store_true",
                    help="one JSON line with the d = 2^16..2^30 sweep instead of the bench line")
    ap.add_argument("--nat", action="store_true",
                    help="one JSON line timing natural compression (quantize + decode-sum)")
    ap.add_argument("--lq", action="store_true",
                    help="one JSON line with the LQ-SGD log-quantizer timings")
    ap.add_argument("--power", action="store_true",
                    help="one JSON line: the fused pass as a burst and sustained, with the "
                         "SM clock of each segment")
    ap.add_argument("--buckets", action="store_true",
                    help="one JSON line comparing the global scale with per-bucket scales")
    ap.add_argument("--dp", action="store_true",
                    help="one JSON line timing the real data-parallel exchange (one worker per "
                         "rank over NCCL) against an fp32 all-reduce; run under torchrun")
    ap.add_argument("--dp-chunks", type=int, default=4,
                    help="--dp also times the chunked exchange (quantize overlapped with the "
                         "all-reduce) with this many chunks; 1 to skip")
    ap.add_argument("--lqsgd", action="store_true",
                    help="one JSON line with the PowerSGD + log-quantizer step timings")
    ap.add_argument("--lqsgd-mats", type=int, default=synthetic.LQ_WORKLOAD["pairs"],
                    help="matrices per worker for --lqsgd (a smaller case for profiling)")
    ap.add_argument("--lqsgd-rank", type=int, default=None, choices=range(1, 9),
                    help="one rank for --lqsgd instead of 1, 4 and 7")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.workload is None:
        args.workload = MODE_WORKLOAD if (args.buckets or args.nat or args.dp) \
            else DEFAULT_WORKLOAD

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    if args.sweep or args.lq or args.buckets or args.lqsgd or args.nat or args.power:
        if rank == 0:
            fn = (run_sweep if args.sweep else run_lq if args.lq else
                  run_buckets if args.buckets else run_nat if args.nat else
                  run_power if args.power else run_lqsgd)
            print(json.dumps(fn(args)), flush=True)
        return

    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    if args.dp:
        store_dir = None
        if world == 1:
            import datetime
            import tempfile
            torch.cuda.set_device(local_rank)
            # a one-rank group: its rendezvous is a file store (no TCP port)
            store_dir = tempfile.mkdtemp(prefix="gq_bench_")
            torch.distributed.init_process_group(
                "nccl", rank=0, world_size=1, init_method="file://" + store_dir + "/store",
                timeout=datetime.timedelta(seconds=120),
                device_id=torch.device("cuda", local_rank))
        try:
            res = run_dp(args, rank, world, local_rank)
            if rank == 0:
                print(json.dumps(res), flush=True)
        finally:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()
            if store_dir is not None:
                import shutil
                shutil.rmtree(store_dir, ignore_errors=True)
        return
    try:
        result = run_ours(args, rank, world, local_rank)
        if rank == 0:
            cpu = not (args.no_cpu_baseline or world > 1)
            # a truncated run (--coords) times the oracle on the same truncation
            sample = args.coords or CPU_SAMPLE_COORDS.get(args.workload)
            result["cpu_baseline"] = cpu_baseline(args.workload, sample) if cpu else None
            result["cpu_baseline_threads"] = \
                cpu_baseline_threads(args.workload, sample) if cpu else None
            if world == 1 and not args.no_extras and not args.coords:
                result["configs"] = run_extras(args, torch.device("cuda", local_rank))
            print(json.dumps(result), flush=True)
    finally:
        if world > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
