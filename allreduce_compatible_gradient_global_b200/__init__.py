"""Python binding of libgq: allreduce-compatible global gradient quantization
on one B200 (sm_100a).

A thin ctypes layer over the C ABI in ``include/gq_api.h``: every function has
the C entry point's name, takes torch tensors (device memory and streams come
from PyTorch), checks dtypes and shapes, passes raw pointers and raises
``GQError`` on a non-zero status.  All arithmetic runs in the CUDA kernels of
libgq.so; there is no fallback: if the library is missing, the first call
raises ImportError with instructions to build it (importing the package alone
does not load it, so that the build step can run from a fresh checkout).
"""
import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgq.so")

GQ_OK = 0
GQ_ERR_ARG = -1
GQ_ERR_OVERFLOW = -2
GQ_ERR_ALIGN = -3
GQ_ERR_CUDA = -4
GQ_ERR_NONFINITE = -5
GQ_ERR_SIZE = -6
GQ_ERR_TIMEOUT = -7

UNIFORM, EXP, LOG, NAT = 0, 1, 2, 3
SCALE_L2, SCALE_MAXABS = 0, 1
WIRE_INT8, WIRE_INT16, WIRE_F16 = 1, 2, 3

_LEVELS = {"uniform": UNIFORM, "exp": EXP, "log": LOG, "nat": NAT}
_SCALES = {"l2": SCALE_L2, "maxabs": SCALE_MAXABS}
_WIRES = {"int8": WIRE_INT8, "int16": WIRE_INT16, "f16": WIRE_F16}


class GQError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__(f"{what}: {gq_status_string(status)} (status {status})")


class _Config(ctypes.Structure):
    _fields_ = [("levels", ctypes.c_int), ("s", ctypes.c_int), ("L", ctypes.c_int),
                ("bits", ctypes.c_int), ("scale_kind", ctypes.c_int), ("wire", ctypes.c_int),
                ("ef", ctypes.c_int), ("alpha", ctypes.c_float),
                ("seed", ctypes.c_ulonglong), ("step", ctypes.c_uint),
                ("worker0", ctypes.c_uint), ("coord0", ctypes.c_ulonglong),
                ("step_dev", ctypes.c_void_p)]


@dataclass
class GQConfig:
    """Mirror of ``gq_config``.  String forms are accepted for the enums."""
    levels: object = "uniform"
    s: int = 15
    L: int = 8
    bits: int = 5
    scale_kind: object = "l2"
    wire: object = "int8"
    ef: bool = False
    alpha: float = 10.0
    seed: int = 0
    step: int = 0
    worker0: int = 0
    coord0: int = 0
    step_dev: object = None  # a CUDA uint32 / int32 tensor of one element, or None

    def c(self) -> _Config:
        lv = _LEVELS.get(self.levels, self.levels)
        sk = _SCALES.get(self.scale_kind, self.scale_kind)
        wr = _WIRES.get(self.wire, self.wire)
        return _Config(int(lv), int(self.s), int(self.L), int(self.bits), int(sk), int(wr),
                       1 if self.ef else 0, float(self.alpha),
                       int(self.seed) & 0xFFFFFFFFFFFFFFFF, int(self.step) & 0xFFFFFFFF,
                       int(self.worker0) & 0xFFFFFFFF, int(self.coord0) & 0xFFFFFFFFFFFFFFFF,
                       None if self.step_dev is None else self.step_dev.data_ptr())

    @property
    def wire_dtype(self):
        wr = _WIRES.get(self.wire, self.wire)
        return {WIRE_INT8: torch.int8, WIRE_INT16: torch.int16, WIRE_F16: torch.float16}[wr]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with "
            "`python -m allreduce_compatible_gradient_global_b200.build` "
            "(or __graft_entry__.build()); there is no CPU fallback")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, LL = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong
    CP = ctypes.POINTER(_Config)
    sig = {
        "gq_version": ([], I),
        "gq_status_string": ([I], ctypes.c_char_p),
        "gq_validate": ([CP, I, LL], I),
        "gq_packed_row_bytes": ([CP, LL, ctypes.POINTER(LL)], I),
        "gq_workspace_bytes": ([CP, I, LL, ctypes.POINTER(ctypes.c_size_t)], I),
        "gq_workspace_init": ([P, ctypes.c_size_t, P], I),
        "gq_get_device_status": ([P, P], I),
        "gq_selftest_wait_timeout": ([P, ctypes.c_uint, P], I),
        "gq_selftest_fma_div": ([P, ctypes.c_float, P, LL, P], I),
        "gq_global_norm": ([P, P, I, LL, CP, P, P, P, P], I),
        "gq_global_norm_noalloc": ([P, P, I, LL, CP, P, P, P], I),
        "gq_quantize_pack": ([P, P, I, LL, CP, P, P, P, P], I),
        "gq_aggregate": ([P, I, LL, CP, P, P, P], I),
        "gq_dequantize_ef": ([P, P, P, P, I, LL, CP, P, P, P, P], I),
        "gq_quantize_aggregate": ([P, P, I, LL, CP, P, P, P, P, P, P], I),
        "gq_step_fused": ([P, P, I, LL, CP, P, P, P, P, P, P, P], I),
        "gq_step_fused_host": ([P, P, P, I, LL, CP, P, P, P, P, P, P, P, P], I),
        "gq_advance_step": ([P, ctypes.c_uint, P], I),
        "gq_bucket_count": ([LL, I, ctypes.POINTER(LL)], I),
        "gq_bucket_workspace_bytes": ([CP, I, LL, I, ctypes.POINTER(ctypes.c_size_t)], I),
        "gq_bucket_scales": ([P, P, I, LL, I, CP, P, P, P], I),
        "gq_quantize_aggregate_bucketed": ([P, P, I, LL, I, CP, P, P, P, P, P, P], I),
        "gq_step_bucketed": ([P, P, I, LL, I, CP, P, P, P, P, P, P], I),
        "gq_psgd_workspace_bytes": ([I, I, P, P, I, ctypes.POINTER(ctypes.c_size_t)], I),
        "gq_psgd_project": ([P, P, I, I, P, P, I, I, P, P, P, P], I),
        "gq_psgd_orthonormalize": ([P, I, P, I, P], I),
        "gq_psgd_back_project": ([P, P, I, I, P, P, I, P, P, P], I),
        "gq_psgd_mean": ([P, P, LL, I, P], I),
        "gq_psgd_reconstruct": ([P, P, I, P, P, I, P, P], I),
        "gq_lqsgd_step": ([P, P, I, I, P, P, I, I, CP, P, P, P, P, P], I),
        "gq_logq_quantize": ([P, I, I, P, P, CP, P, P, P, P], I),
        "gq_logq_decode_sum": ([P, P, I, I, P, P, CP, P, P], I),
        "gq_nat_quantize": ([P, I, LL, CP, P, P, P], I),
        "gq_nat_decode_sum": ([P, I, LL, P, P], I),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


_lib = None


def lib():
    """The loaded libgq.so (loaded on first use; raises if it is missing)."""
    global _lib
    if _lib is None:
        _lib = _load()
    return _lib


def gq_version() -> int:
    return lib().gq_version()


def gq_status_string(status: int) -> str:
    return lib().gq_status_string(int(status)).decode()


# ------------------------------------------------------------------ marshalling
def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(rc, what):
    if rc != GQ_OK:
        raise GQError(rc, what)


def _need(t, dtype, shape, name, cuda=True):
    if t is None:
        return
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if cuda and not t.is_cuda:
        raise TypeError(f"{name}: expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")


def _wd(g):
    if g.dim() != 2:
        raise ValueError("gradients must be [W][d]")
    return int(g.shape[0]), int(g.shape[1])


# ------------------------------------------------------------------ sizes
def gq_validate(cfg: GQConfig, W: int, d: int) -> int:
    c = cfg.c()
    return lib().gq_validate(ctypes.byref(c), int(W), int(d))


def gq_packed_row_bytes(cfg: GQConfig, d: int) -> int:
    c = cfg.c()
    out = ctypes.c_longlong()
    _check(lib().gq_packed_row_bytes(ctypes.byref(c), int(d), ctypes.byref(out)),
           "gq_packed_row_bytes")
    return out.value


def gq_workspace_bytes(cfg: GQConfig, W: int, d: int) -> int:
    c = cfg.c()
    out = ctypes.c_size_t()
    _check(lib().gq_workspace_bytes(ctypes.byref(c), int(W), int(d), ctypes.byref(out)),
           "gq_workspace_bytes")
    return out.value


def gq_workspace_init(ws, stream=None):
    _check(lib().gq_workspace_init(_ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "gq_workspace_init")


def gq_get_device_status(ws, stream=None) -> int:
    """Synchronizes the stream; returns GQ_OK or GQ_ERR_NONFINITE (and clears the
    flag).  A timed-out pipeline wait raises GQError(GQ_ERR_TIMEOUT)."""
    rc = lib().gq_get_device_status(_ptr(ws), _stream(stream))
    if rc not in (GQ_OK, GQ_ERR_NONFINITE):
        raise GQError(rc, "gq_get_device_status")
    return rc


def gq_selftest_wait_timeout(ws, limit_ms=50, stream=None):
    """Make one bounded device wait expire on purpose; returns the status that
    gq_get_device_status then reports (GQ_ERR_TIMEOUT when detection works)."""
    _check(lib().gq_selftest_wait_timeout(_ptr(ws), int(limit_ms), _stream(stream)),
           "gq_selftest_wait_timeout")
    return lib().gq_get_device_status(_ptr(ws), _stream(stream))


def gq_selftest_fma_div(a, b, out, stream=None):
    """out = a / b as the log quantizer divides (see gq_api.h); a, out: float32
    CUDA tensors of one shape, b a positive finite float."""
    _need(a, torch.float32, tuple(a.shape), "a")
    _need(out, torch.float32, tuple(a.shape), "out")
    _check(lib().gq_selftest_fma_div(_ptr(a), float(b), _ptr(out), a.numel(), _stream(stream)),
           "gq_selftest_fma_div")


def gq_advance_step(step_dev, by=1, stream=None):
    """step_dev[0] += by on the stream (the device step counter of a captured
    step graph; see GQConfig.step_dev)."""
    _need(step_dev, step_dev.dtype, (1,), "step_dev")
    if step_dev.element_size() != 4:
        raise TypeError("step_dev: a 32-bit integer tensor")
    _check(lib().gq_advance_step(_ptr(step_dev), int(by), _stream(stream)), "gq_advance_step")


# ------------------------------------------------------------------ the path
def gq_global_norm(g, e, cfg: GQConfig, scale, norms, ws, stream=None):
    W, d = _wd(g)
    _need(g, torch.float32, (W, d), "g")
    _need(e, torch.float32, (W, d), "e")
    _need(scale, torch.float32, (1,), "scale")
    _need(norms, torch.float64, (W,), "norms")
    c = cfg.c()
    _check(lib().gq_global_norm(_ptr(g), _ptr(e), W, d, ctypes.byref(c), _ptr(scale), _ptr(norms),
                               _ptr(ws), _stream(stream)), "gq_global_norm")


def gq_global_norm_noalloc(g, e, cfg: GQConfig, scale, norms, stream=None):
    """gq_global_norm without a workspace, for callers that cannot allocate:
    the library's own fixed device scratch holds the partial sums (W <= 4096;
    calls that overlap on the GPU race on that scratch)."""
    W, d = _wd(g)
    _need(g, torch.float32, (W, d), "g")
    _need(e, torch.float32, (W, d), "e")
    _need(scale, torch.float32, (1,), "scale")
    _need(norms, torch.float64, (W,), "norms")
    c = cfg.c()
    _check(lib().gq_global_norm_noalloc(_ptr(g), _ptr(e), W, d, ctypes.byref(c), _ptr(scale),
                                       _ptr(norms), _stream(stream)), "gq_global_norm_noalloc")


def gq_quantize_pack(g, e, cfg: GQConfig, scale, codes, ws, stream=None):
    W, d = _wd(g)
    _need(g, torch.float32, (W, d), "g")
    _need(e, torch.float32, (W, d), "e")
    _need(codes, torch.uint8, (W, gq_packed_row_bytes(cfg, d)), "codes")
    c = cfg.c()
    _check(lib().gq_quantize_pack(_ptr(g), _ptr(e), W, d, ctypes.byref(c), _ptr(scale),
                                 _ptr(codes), _ptr(ws), _stream(stream)), "gq_quantize_pack")


def gq_aggregate(codes, W, d, cfg: GQConfig, sum_out, ws, stream=None):
    _need(codes, torch.uint8, (W, gq_packed_row_bytes(cfg, d)), "codes")
    _need(sum_out, cfg.wire_dtype, (d,), "sum")
    c = cfg.c()
    _check(lib().gq_aggregate(_ptr(codes), int(W), int(d), ctypes.byref(c), _ptr(sum_out),
                             _ptr(ws), _stream(stream)), "gq_aggregate")


def gq_dequantize_ef(sum_in, codes, g, e, W, d, cfg: GQConfig, scale, out, ws, stream=None):
    _need(sum_in, cfg.wire_dtype, (d,), "sum")
    _need(codes, torch.uint8, (W, gq_packed_row_bytes(cfg, d)), "codes")
    _need(g, torch.float32, (W, d), "g")
    _need(e, torch.float32, (W, d), "e")
    _need(out, torch.float32, (d,), "out")
    c = cfg.c()
    _check(lib().gq_dequantize_ef(_ptr(sum_in), _ptr(codes), _ptr(g), _ptr(e), int(W), int(d),
                                 ctypes.byref(c), _ptr(scale), _ptr(out), _ptr(ws),
                                 _stream(stream)), "gq_dequantize_ef")


def gq_quantize_aggregate(g, e, cfg: GQConfig, scale, codes, sum_out, out, ws, stream=None):
    W, d = _wd(g)
    _need(g, torch.float32, (W, d), "g")
    _need(e, torch.float32, (W, d), "e")
    _need(codes, torch.uint8, (W, gq_packed_row_bytes(cfg, d)), "codes")
    _need(sum_out, cfg.wire_dtype, (d,), "sum")
    _need(out, torch.float32, (d,), "out")
    c = cfg.c()
    _check(lib().gq_quantize_aggregate(_ptr(g), _ptr(e), W, d, ctypes.byref(c), _ptr(scale),
                                      _ptr(codes), _ptr(sum_out), _ptr(out), _ptr(ws),
                                      _stream(stream)), "gq_quantize_aggregate")


def gq_step_fused(g, e, cfg: GQConfig, scale, norms, codes, sum_out, out, ws, stream=None):
    W, d = _wd(g)
    _need(g, torch.float32, (W, d), "g")
    _need(e, torch.float32, (W, d), "e")
    _need(scale, torch.float32, (1,), "scale")
    _need(norms, torch.float64, (W,), "norms")
    _need(codes, torch.uint8, (W, gq_packed_row_bytes(cfg, d)), "codes")
    _need(sum_out, cfg.wire_dtype, (d,), "sum")
    _need(out, torch.float32, (d,), "out")
    c = cfg.c()
    _check(lib().gq_step_fused(_ptr(g), _ptr(e), W, d, ctypes.byref(c), _ptr(scale), _ptr(norms),
                              _ptr(codes), _ptr(sum_out), _ptr(out), _ptr(ws), _stream(stream)),
           "gq_step_fused")


def gq_step_fused_host(g_host, g_dev, e, cfg: GQConfig, scale, codes, sum_out, out, out_host,
                       scale_host, ws, stream=None):
    """g_host / out_host / scale_host: CPU tensors (pinned for full speed)."""
    W, d = _wd(g_dev)
    _need(g_host, torch.float32, (W, d), "g_host", cuda=False)
    _need(out_host, torch.float32, (d,), "out_host", cuda=False)
    _need(scale_host, torch.float32, (1,), "scale_host", cuda=False)
    _need(g_dev, torch.float32, (W, d), "g_dev")
    _need(out, torch.float32, (d,), "out")
    c = cfg.c()
    _check(lib().gq_step_fused_host(_ptr(g_host), _ptr(g_dev), _ptr(e), W, d, ctypes.byref(c),
                                   _ptr(scale), _ptr(codes), _ptr(sum_out), _ptr(out),
                                   _ptr(out_host), _ptr(scale_host), _ptr(ws), _stream(stream)),
           "gq_step_fused_host")


def _shapes(rows, cols):
    r = (ctypes.c_int * len(rows))(*[int(x) for x in rows])
    c = (ctypes.c_int * len(cols))(*[int(x) for x in cols])
    return r, c


def gq_logq_quantize(x, rows, cols, cfg: GQConfig, maxabs, codes, ws, stream=None):
    W, n = _wd(x)
    if len(rows) != len(cols) or sum(int(a) * int(b) for a, b in zip(rows, cols)) != n:
        raise ValueError("rows/cols do not add up to the factor buffer")
    _need(x, torch.float32, (W, n), "x")
    _need(maxabs, torch.float32, (W, len(rows)), "maxabs")
    _need(codes, torch.int8, (W, n), "codes")
    r, cc = _shapes(rows, cols)
    c = cfg.c()
    _check(lib().gq_logq_quantize(_ptr(x), W, len(rows), r, cc, ctypes.byref(c), _ptr(maxabs),
                                 _ptr(codes), _ptr(ws), _stream(stream)), "gq_logq_quantize")


def gq_logq_decode_sum(codes, maxabs, rows, cols, cfg: GQConfig, out, stream=None):
    W, n = _wd(codes)
    _need(codes, torch.int8, (W, n), "codes")
    _need(maxabs, torch.float32, (W, len(rows)), "maxabs")
    _need(out, torch.float32, (n,), "out")
    r, cc = _shapes(rows, cols)
    c = cfg.c()
    _check(lib().gq_logq_decode_sum(_ptr(codes), _ptr(maxabs), W, len(rows), r, cc,
                                   ctypes.byref(c), _ptr(out), _stream(stream)),
           "gq_logq_decode_sum")


# ------------------------------------------------------------------ natural compression
def gq_nat_quantize(x, cfg: GQConfig, codes, ws, stream=None):
    """x [W][n] fp32 -> codes [W][n] int16 (sign << 8 | exponent of the signed power
    of two); cfg.levels == "nat" (seed, step / step_dev and worker0 are used)."""
    W, n = _wd(x)
    _need(x, torch.float32, (W, n), "x")
    _need(codes, torch.int16, (W, n), "codes")
    c = cfg.c()
    _check(lib().gq_nat_quantize(_ptr(x), W, n, ctypes.byref(c), _ptr(codes), _ptr(ws),
                                 _stream(stream)), "gq_nat_quantize")


def gq_nat_decode_sum(codes, out, stream=None):
    """codes [W][n] int16 -> out [n] fp32, the values summed over workers in
    ascending order."""
    W, n = _wd(codes)
    _need(codes, torch.int16, (W, n), "codes")
    _need(out, torch.float32, (n,), "out")
    _check(lib().gq_nat_decode_sum(_ptr(codes), W, n, _ptr(out), _stream(stream)),
           "gq_nat_decode_sum")


# ------------------------------------------------------------------ per-bucket scales
def gq_bucket_count(d: int, bucket_log2: int) -> int:
    out = ctypes.c_longlong()
    _check(lib().gq_bucket_count(int(d), int(bucket_log2), ctypes.byref(out)), "gq_bucket_count")
    return out.value


def gq_bucket_workspace_bytes(cfg: GQConfig, W: int, d: int, bucket_log2: int) -> int:
    c = cfg.c()
    out = ctypes.c_size_t()
    _check(lib().gq_bucket_workspace_bytes(ctypes.byref(c), int(W), int(d), int(bucket_log2),
                                           ctypes.byref(out)), "gq_bucket_workspace_bytes")
    return out.value


def gq_bucket_scales(g, e, bucket_log2, cfg: GQConfig, table, ws, stream=None):
    """table: float32 [3 * K] = S_k | multipliers | units."""
    W, d = _wd(g)
    _need(g, torch.float32, (W, d), "g")
    _need(e, torch.float32, (W, d), "e")
    _need(table, torch.float32, (3 * gq_bucket_count(d, bucket_log2),), "table")
    c = cfg.c()
    _check(lib().gq_bucket_scales(_ptr(g), _ptr(e), W, d, int(bucket_log2), ctypes.byref(c),
                                  _ptr(table), _ptr(ws), _stream(stream)), "gq_bucket_scales")


def gq_quantize_aggregate_bucketed(g, e, bucket_log2, cfg: GQConfig, table, codes, sum_out, out,
                                   ws, stream=None):
    W, d = _wd(g)
    _need(g, torch.float32, (W, d), "g")
    _need(e, torch.float32, (W, d), "e")
    _need(table, torch.float32, (3 * gq_bucket_count(d, bucket_log2),), "table")
    _need(codes, torch.uint8, (W, gq_packed_row_bytes(cfg, d)), "codes")
    _need(sum_out, cfg.wire_dtype, (d,), "sum")
    _need(out, torch.float32, (d,), "out")
    c = cfg.c()
    _check(lib().gq_quantize_aggregate_bucketed(
        _ptr(g), _ptr(e), W, d, int(bucket_log2), ctypes.byref(c), _ptr(table), _ptr(codes),
        _ptr(sum_out), _ptr(out), _ptr(ws), _stream(stream)), "gq_quantize_aggregate_bucketed")


def gq_step_bucketed(g, e, bucket_log2, cfg: GQConfig, table, codes, sum_out, out, ws,
                     stream=None):
    W, d = _wd(g)
    _need(g, torch.float32, (W, d), "g")
    _need(e, torch.float32, (W, d), "e")
    _need(table, torch.float32, (3 * gq_bucket_count(d, bucket_log2),), "table")
    _need(codes, torch.uint8, (W, gq_packed_row_bytes(cfg, d)), "codes")
    _need(sum_out, cfg.wire_dtype, (d,), "sum")
    _need(out, torch.float32, (d,), "out")
    c = cfg.c()
    _check(lib().gq_step_bucketed(_ptr(g), _ptr(e), W, d, int(bucket_log2), ctypes.byref(c),
                                  _ptr(table), _ptr(codes), _ptr(sum_out), _ptr(out), _ptr(ws),
                                  _stream(stream)), "gq_step_bucketed")


# ------------------------------------------------------------------ PowerSGD + LQ
class PsgdShapes:
    """The matrices of one worker: rows[l] x cols[l], and the rank."""

    def __init__(self, rows, cols, rank):
        if len(rows) != len(cols):
            raise ValueError("rows and cols differ in length")
        self.rows = [int(x) for x in rows]
        self.cols = [int(x) for x in cols]
        self.rank = int(rank)
        self._r = (ctypes.c_int * len(self.rows))(*self.rows)
        self._c = (ctypes.c_int * len(self.cols))(*self.cols)

    @property
    def nmats(self):
        return len(self.rows)

    @property
    def total(self):
        return sum(n * m for n, m in zip(self.rows, self.cols))

    @property
    def ptotal(self):
        return sum(self.rows) * self.rank

    @property
    def qtotal(self):
        return sum(self.cols) * self.rank


def gq_psgd_workspace_bytes(W: int, sh: PsgdShapes) -> int:
    out = ctypes.c_size_t()
    _check(lib().gq_psgd_workspace_bytes(int(W), sh.nmats, sh._r, sh._c, sh.rank,
                                         ctypes.byref(out)), "gq_psgd_workspace_bytes")
    return out.value


def gq_psgd_project(g, m, sh: PsgdShapes, have_prev, p_prev, q, pw, stream=None):
    W = int(g.shape[0])
    _need(g, torch.float32, (W, sh.total), "g")
    _need(m, torch.float32, (W, sh.total), "m")
    _need(p_prev, torch.float32, (sh.ptotal,), "p_prev")
    _need(q, torch.float32, (sh.qtotal,), "q")
    _need(pw, torch.float32, (W, sh.ptotal), "pw")
    _check(lib().gq_psgd_project(_ptr(g), _ptr(m), W, sh.nmats, sh._r, sh._c, sh.rank,
                                 1 if have_prev else 0, _ptr(p_prev), _ptr(q), _ptr(pw),
                                 _stream(stream)), "gq_psgd_project")


def gq_psgd_orthonormalize(p, sh: PsgdShapes, stream=None):
    _need(p, torch.float32, (sh.ptotal,), "p")
    _check(lib().gq_psgd_orthonormalize(_ptr(p), sh.nmats, sh._r, sh.rank, _stream(stream)),
           "gq_psgd_orthonormalize")


def gq_psgd_back_project(m, p, sh: PsgdShapes, qw, ws, stream=None):
    W = int(m.shape[0])
    _need(m, torch.float32, (W, sh.total), "m")
    _need(p, torch.float32, (sh.ptotal,), "p")
    _need(qw, torch.float32, (W, sh.qtotal), "qw")
    _check(lib().gq_psgd_back_project(_ptr(m), _ptr(p), W, sh.nmats, sh._r, sh._c, sh.rank,
                                      _ptr(qw), _ptr(ws), _stream(stream)), "gq_psgd_back_project")


def gq_psgd_mean(sum_in, out, W, stream=None):
    _need(sum_in, torch.float32, None, "sum")
    _need(out, torch.float32, tuple(sum_in.shape), "out")
    _check(lib().gq_psgd_mean(_ptr(sum_in), _ptr(out), sum_in.numel(), int(W), _stream(stream)),
           "gq_psgd_mean")


def gq_psgd_reconstruct(p, q, sh: PsgdShapes, ghat, stream=None):
    _need(p, torch.float32, (sh.ptotal,), "p")
    _need(q, torch.float32, (sh.qtotal,), "q")
    _need(ghat, torch.float32, (sh.total,), "ghat")
    _check(lib().gq_psgd_reconstruct(_ptr(p), _ptr(q), sh.nmats, sh._r, sh._c, sh.rank,
                                     _ptr(ghat), _stream(stream)), "gq_psgd_reconstruct")


def gq_lqsgd_step(g, m, sh: PsgdShapes, have_prev, cfg: GQConfig, p, q, ghat, ws, stream=None):
    W = int(g.shape[0])
    _need(g, torch.float32, (W, sh.total), "g")
    _need(m, torch.float32, (W, sh.total), "m")
    _need(p, torch.float32, (sh.ptotal,), "p")
    _need(q, torch.float32, (sh.qtotal,), "q")
    _need(ghat, torch.float32, (sh.total,), "ghat")
    c = cfg.c()
    _check(lib().gq_lqsgd_step(_ptr(g), _ptr(m), W, sh.nmats, sh._r, sh._c, sh.rank,
                               1 if have_prev else 0, ctypes.byref(c), _ptr(p), _ptr(q),
                               _ptr(ghat), _ptr(ws), _stream(stream)), "gq_lqsgd_step")


# ------------------------------------------------------------------ buffers
class StepBuffers:
    """Device buffers of one step for W workers and d coordinates."""

    def __init__(self, cfg: GQConfig, W: int, d: int, device="cuda", codes=True, ef=None):
        self.cfg, self.W, self.d = cfg, W, d
        ef = cfg.ef if ef is None else ef
        self.scale = torch.zeros(1, dtype=torch.float32, device=device)
        self.norms = torch.zeros(W, dtype=torch.float64, device=device)
        self.codes = (torch.empty((W, gq_packed_row_bytes(cfg, d)), dtype=torch.uint8,
                                  device=device) if codes else None)
        self.sum = torch.empty(d, dtype=cfg.wire_dtype, device=device)
        self.out = torch.empty(d, dtype=torch.float32, device=device)
        self.e = torch.zeros((W, d), dtype=torch.float32, device=device) if ef else None
        nbytes = gq_workspace_bytes(cfg, W, d)
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
        gq_workspace_init(self.ws)
