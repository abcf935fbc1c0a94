"""The C ABI without a GPU: the library builds, loads, exports every entry point
that include/gq_api.h declares, and its host-side checks (sizes, overflow
rule, alignment) answer before anything is launched."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gq_api.h")


def declared_entry_points():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"GQ_API\s+[\w\s\*]+?\b(gq_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def gq():
    from allreduce_compatible_gradient_global_b200 import build as b
    b.build()
    import allreduce_compatible_gradient_global_b200 as gq
    return gq


def test_header_declares_the_path():
    names = declared_entry_points()
    for required in ("gq_global_norm", "gq_quantize_pack", "gq_aggregate", "gq_dequantize_ef",
                     "gq_step_fused", "gq_quantize_aggregate", "gq_step_fused_host",
                     "gq_logq_quantize", "gq_logq_decode_sum", "gq_workspace_bytes"):
        assert required in names


def test_library_exports_every_declared_symbol(gq):
    names = declared_entry_points()
    nm = subprocess.run(["nm", "-D", "--defined-only", gq.LIB_PATH], capture_output=True,
                        text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(gq_\w+)$", nm, flags=re.M))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    lib = ctypes.CDLL(gq.LIB_PATH)
    for n in names:
        assert getattr(lib, n) is not None


def test_division_selftest_checks_its_arguments_on_the_host(gq):
    lib = gq.lib()
    for b in (0.0, -1.0, float("inf"), float("nan")):
        assert lib.gq_selftest_fma_div(None, b, None, 0, None) == gq.GQ_ERR_ARG
    assert lib.gq_selftest_fma_div(None, 2.0, None, 0, None) == gq.GQ_OK  # nothing to do
    assert lib.gq_selftest_fma_div(None, 2.0, None, 5, None) == gq.GQ_ERR_ARG


def test_version_and_status_strings(gq):
    assert gq.gq_version() >= 100
    for st in (0, -1, -2, -3, -4, -5, -6, -7):
        assert gq.gq_status_string(st) != "unknown status"


def cfg(gq, **kw):
    return gq.GQConfig(**kw)


def test_overflow_rule(gq):
    # uniform: W * s must fit the sum type
    assert gq.gq_validate(cfg(gq, s=15, bits=5, wire="int8"), 8, 100) == gq.GQ_OK      # 120
    assert gq.gq_validate(cfg(gq, s=15, bits=5, wire="int8"), 9, 100) == gq.GQ_ERR_OVERFLOW
    assert gq.gq_validate(cfg(gq, s=127, bits=8, wire="int16"), 8, 100) == gq.GQ_OK
    assert gq.gq_validate(cfg(gq, s=127, bits=8, wire="int8"), 2, 100) == gq.GQ_ERR_OVERFLOW
    # exponential: sums count 2^(L-1) units of the finest level per worker
    assert gq.gq_validate(cfg(gq, levels="exp", L=8, bits=5, wire="int16"), 8, 10) == gq.GQ_OK
    assert gq.gq_validate(cfg(gq, levels="exp", L=8, bits=5, wire="int8"), 1, 10) == \
        gq.GQ_ERR_OVERFLOW                                                             # 128
    assert gq.gq_validate(cfg(gq, levels="exp", L=7, bits=4, wire="int8"), 1, 10) == gq.GQ_OK
    assert gq.gq_validate(cfg(gq, levels="exp", L=7, bits=4, wire="int8"), 2, 10) == \
        gq.GQ_ERR_OVERFLOW
    assert gq.gq_validate(cfg(gq, levels="exp", L=15, bits=5, wire="int16"), 1, 10) == gq.GQ_OK
    assert gq.gq_validate(cfg(gq, levels="exp", L=15, bits=5, wire="int16"), 2, 10) == \
        gq.GQ_ERR_OVERFLOW


def test_bits_must_hold_the_codes(gq):
    assert gq.gq_validate(cfg(gq, s=7, bits=4, wire="int8"), 1, 10) == gq.GQ_OK
    assert gq.gq_validate(cfg(gq, s=8, bits=4, wire="int8"), 1, 10) == gq.GQ_ERR_ARG
    assert gq.gq_validate(cfg(gq, s=15, bits=5, wire="int8"), 1, 10) == gq.GQ_OK
    assert gq.gq_validate(cfg(gq, s=16, bits=5, wire="int8"), 1, 10) == gq.GQ_ERR_ARG
    assert gq.gq_validate(cfg(gq, s=127, bits=8, wire="int8"), 1, 10) == gq.GQ_OK
    assert gq.gq_validate(cfg(gq, s=128, bits=8, wire="int16"), 1, 10) == gq.GQ_ERR_ARG
    assert gq.gq_validate(cfg(gq, levels="exp", L=7, bits=4, wire="int16"), 1, 10) == gq.GQ_OK
    assert gq.gq_validate(cfg(gq, levels="exp", L=8, bits=4, wire="int16"), 1, 10) == \
        gq.GQ_ERR_ARG
    assert gq.gq_validate(cfg(gq, bits=6), 1, 10) == gq.GQ_ERR_ARG


def test_bad_levels_and_sizes(gq):
    assert gq.gq_validate(cfg(gq, s=0), 1, 10) == gq.GQ_ERR_ARG
    assert gq.gq_validate(cfg(gq, levels="exp", L=0), 1, 10) == gq.GQ_ERR_ARG
    assert gq.gq_validate(cfg(gq, levels="exp", L=16, bits=16, wire="int16"), 1, 10) == \
        gq.GQ_ERR_ARG
    assert gq.gq_validate(cfg(gq, levels=7), 1, 10) == gq.GQ_ERR_ARG
    assert gq.gq_validate(cfg(gq, scale_kind=5), 1, 10) == gq.GQ_ERR_ARG
    assert gq.gq_validate(cfg(gq, wire=4), 1, 10) == gq.GQ_ERR_ARG
    assert gq.gq_validate(cfg(gq, wire=0), 1, 10) == gq.GQ_ERR_ARG
    assert gq.gq_validate(cfg(gq), 0, 10) == gq.GQ_ERR_ARG
    assert gq.gq_validate(cfg(gq), 1, -1) == gq.GQ_ERR_ARG
    assert gq.gq_validate(cfg(gq), 1, 0) == gq.GQ_OK


def test_packed_row_bytes_and_workspace(gq):
    for bits in (4, 5, 8, 16):
        for d in (0, 1, 127, 128, 129, 25_557_032, 1 << 30):
            assert gq.gq_packed_row_bytes(cfg(gq, bits=bits), d) == -(-d // 128) * 16 * bits
    ws = gq.gq_workspace_bytes(cfg(gq), 8, 1 << 20)
    assert ws >= 256 + 8 * 8 and ws % 16 == 0


def test_entry_points_reject_before_launch(gq):
    lib = gq.lib()
    c = cfg(gq, s=15, bits=5, wire="int8").c()
    P = ctypes.c_void_p
    good = P(0x10000000)
    odd = P(0x10000004)
    # null / bad sizes
    assert lib.gq_global_norm(None, None, 4, 100, ctypes.byref(c), good, None, good, None) == \
        gq.GQ_ERR_ARG
    assert lib.gq_global_norm(good, None, 0, 100, ctypes.byref(c), good, None, good, None) == \
        gq.GQ_ERR_ARG
    # misaligned gradient
    assert lib.gq_global_norm(odd, None, 4, 100, ctypes.byref(c), good, None, good, None) == \
        gq.GQ_ERR_ALIGN
    # overflowing wire type is caught before the quantize launch
    assert lib.gq_quantize_aggregate(good, None, 9, 100, ctypes.byref(c), good, good, good, good,
                                     good, None) == gq.GQ_ERR_OVERFLOW
    # EF requested without an error buffer
    cef = cfg(gq, s=15, bits=5, wire="int8", ef=True).c()
    assert lib.gq_step_fused(good, None, 4, 100, ctypes.byref(cef), good, None, good, good, good,
                             good, None) == gq.GQ_ERR_ARG
    # nothing requested
    assert lib.gq_quantize_aggregate(good, None, 4, 100, ctypes.byref(c), good, None, None, None,
                                     good, None) == gq.GQ_ERR_ARG
    # LQ calls need the LOG level set and matching shapes
    rows = (ctypes.c_int * 2)(4096, 4096)
    cols = (ctypes.c_int * 2)(1, 1)
    assert lib.gq_logq_quantize(good, 8, 2, rows, cols, ctypes.byref(c), good, good, good,
                                None) == gq.GQ_ERR_ARG
    clog = cfg(gq, levels="log", alpha=10.0).c()
    assert lib.gq_logq_quantize(good, 8, 0, rows, cols, ctypes.byref(clog), good, good, good,
                                None) == gq.GQ_ERR_ARG
    clog_bad = cfg(gq, levels="log", alpha=-1.0).c()
    assert lib.gq_logq_decode_sum(good, good, 8, 2, rows, cols, ctypes.byref(clog_bad), good,
                                  None) == gq.GQ_ERR_ARG


def test_bucket_sizes_and_workspace(gq):
    assert gq.gq_bucket_count(0, 10) == 0
    assert gq.gq_bucket_count(1024, 10) == 1
    assert gq.gq_bucket_count(1025, 10) == 2
    assert gq.gq_bucket_count(25_557_032, 17) == -(-25_557_032 // (1 << 17))
    assert gq.gq_bucket_count(1 << 30, 30) == 1
    for bad in (6, 31, -1):
        with pytest.raises(gq.GQError):
            gq.gq_bucket_count(100, bad)
    c = cfg(gq)
    for W, d, b in ((8, 25_557_032, 17), (1, 100, 7), (8, 1 << 30, 12), (40, 8192, 10)):
        n = gq.gq_bucket_workspace_bytes(c, W, d, b)
        chunks = -(-d // (1 << min(b, 12)))
        assert n >= 256 + W * chunks * 12
        assert n >= gq.gq_workspace_bytes(c, W, d)  # also a valid global-path workspace
        assert n % 256 == 0


def test_bucket_entry_points_reject_before_launch(gq):
    lib = gq.lib()
    c = cfg(gq, s=15, bits=5, wire="int8").c()
    P = ctypes.c_void_p
    good = P(0x10000000)
    odd = P(0x10000004)
    assert lib.gq_bucket_scales(good, None, 4, 4096, 6, ctypes.byref(c), good, good, None) == \
        gq.GQ_ERR_ARG
    assert lib.gq_bucket_scales(odd, None, 4, 4096, 10, ctypes.byref(c), good, good, None) == \
        gq.GQ_ERR_ALIGN
    assert lib.gq_bucket_scales(good, None, 4, 4096, 10, ctypes.byref(c), None, good, None) == \
        gq.GQ_ERR_ARG
    assert lib.gq_quantize_aggregate_bucketed(good, None, 9, 4096, 10, ctypes.byref(c), good,
                                              good, good, good, good, None) == \
        gq.GQ_ERR_OVERFLOW
    cef = cfg(gq, s=15, bits=5, wire="int8", ef=True).c()
    assert lib.gq_step_bucketed(good, None, 4, 4096, 10, ctypes.byref(cef), good, good, good,
                                good, good, None) == gq.GQ_ERR_ARG
    clog = cfg(gq, levels="log", alpha=10.0).c()
    assert lib.gq_step_bucketed(good, None, 4, 4096, 10, ctypes.byref(clog), good, good, good,
                                good, good, None) == gq.GQ_ERR_ARG


def test_psgd_entry_points_reject_before_launch(gq):
    lib = gq.lib()
    P = ctypes.c_void_p
    good = P(0x10000000)
    odd = P(0x10000004)
    rows = (ctypes.c_int * 2)(64, 32)
    cols = (ctypes.c_int * 2)(48, 32)
    n = ctypes.c_size_t()
    assert lib.gq_psgd_workspace_bytes(2, 2, rows, cols, 4, ctypes.byref(n)) == gq.GQ_OK
    assert n.value > 256
    for bad_rank in (0, 9):
        assert lib.gq_psgd_workspace_bytes(2, 2, rows, cols, bad_rank, ctypes.byref(n)) == \
            gq.GQ_ERR_ARG
    assert lib.gq_psgd_workspace_bytes(0, 2, rows, cols, 4, ctypes.byref(n)) == gq.GQ_ERR_ARG
    zero = (ctypes.c_int * 1)(0)
    assert lib.gq_psgd_workspace_bytes(2, 1, zero, cols, 4, ctypes.byref(n)) == gq.GQ_ERR_ARG
    # have_prev without a previous P
    assert lib.gq_psgd_project(good, good, 2, 2, rows, cols, 4, 1, None, good, good, None) == \
        gq.GQ_ERR_ARG
    assert lib.gq_psgd_project(odd, good, 2, 2, rows, cols, 4, 0, None, good, good, None) == \
        gq.GQ_ERR_ALIGN
    assert lib.gq_psgd_back_project(good, good, 2, 2, rows, cols, 4, good, None, None) == \
        gq.GQ_ERR_ARG
    assert lib.gq_psgd_mean(good, good, 10, 0, None) == gq.GQ_ERR_ARG
    c = cfg(gq).c()  # not the log level set
    assert lib.gq_lqsgd_step(good, good, 2, 2, rows, cols, 4, 0, ctypes.byref(c), good, good,
                             None, good, None) == gq.GQ_ERR_ARG


def test_workspace_and_config_layout(gq):
    """gq_config carries worker0 and coord0 after step (the C struct and the
    binding agree); coord0 must be a multiple of 4."""
    assert ctypes.sizeof(gq._Config) == 64
    assert gq._Config.step_dev.offset == 56
    assert gq._Config.worker0.offset == 44
    assert gq._Config.coord0.offset == 48
    assert gq.gq_validate(cfg(gq, coord0=4096), 1, 10) == gq.GQ_OK
    assert gq.gq_validate(cfg(gq, coord0=6), 1, 10) == gq.GQ_ERR_ARG


def test_natural_compression_argument_checks(gq):
    """Checked on the host before any launch (nothing here reaches a GPU)."""
    lib = gq.lib()
    good = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 4)
    cnat = cfg(gq, levels="nat", seed=3).c()
    cuni = cfg(gq).c()
    assert lib.gq_nat_quantize(good, 4, 100, ctypes.byref(cuni), good, good, None) == \
        gq.GQ_ERR_ARG                                   # levels must be GQ_NAT
    assert lib.gq_nat_quantize(good, 0, 100, ctypes.byref(cnat), good, good, None) == \
        gq.GQ_ERR_ARG                                   # no workers
    assert lib.gq_nat_quantize(good, 4, -1, ctypes.byref(cnat), good, good, None) == \
        gq.GQ_ERR_ARG
    assert lib.gq_nat_quantize(good, 65536, 4, ctypes.byref(cnat), good, good, None) == \
        gq.GQ_ERR_ARG                                   # one grid row per worker
    assert lib.gq_nat_quantize(good, 4, 100, ctypes.byref(cnat), good, None, None) == \
        gq.GQ_ERR_ARG                                   # no workspace
    assert lib.gq_nat_quantize(odd, 4, 100, ctypes.byref(cnat), good, good, None) == \
        gq.GQ_ERR_ALIGN
    assert lib.gq_nat_quantize(good, 4, 100, ctypes.byref(cnat), odd, good, None) == \
        gq.GQ_ERR_ALIGN
    assert lib.gq_nat_quantize(None, 4, 0, ctypes.byref(cnat), None, good, None) == gq.GQ_OK
    assert lib.gq_nat_decode_sum(good, 0, 100, good, None) == gq.GQ_ERR_ARG
    assert lib.gq_nat_decode_sum(None, 4, 100, good, None) == gq.GQ_ERR_ARG
    assert lib.gq_nat_decode_sum(good, 4, 100, odd, None) == gq.GQ_ERR_ALIGN
    assert lib.gq_nat_decode_sum(None, 4, 0, None, None) == gq.GQ_OK
    # the main path does not take the natural-compression level
    assert gq.gq_validate(gq.GQConfig(levels="nat"), 4, 100) == gq.GQ_ERR_ARG

