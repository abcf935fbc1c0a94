"""ctypes binding of the CPU oracle (TEST INFRASTRUCTURE ONLY).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg import this package.  It restates, slowly and plainly, what the GPU path
computes; it never imports the product package and the product never imports
it.  Every function takes and returns numpy arrays.
"""
import ctypes
import os

import numpy as np

from . import build as _build

UNIFORM, EXP = 0, 1
SCALE_L2, SCALE_MAXABS = 0, 1

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i64, i32, u32, u64, f32 = (ctypes.c_int64, ctypes.c_int, ctypes.c_uint32,
                                   ctypes.c_uint64, ctypes.c_float)
        L.gqo_philox4x32.argtypes = [P, u32, u32, i32]
        L.gqo_philox4x32.restype = None
        L.gqo_uniform_bits.argtypes = [u64, u32, u32, u32, u64]
        L.gqo_uniform_bits.restype = u32
        L.gqo_sumsq.argtypes = [P, P, i64]
        L.gqo_sumsq.restype = ctypes.c_double
        L.gqo_sumsq_from.argtypes = [ctypes.c_double, P, P, i64]
        L.gqo_sumsq_from.restype = ctypes.c_double
        L.gqo_maxabs.argtypes = [P, P, i64]
        L.gqo_maxabs.restype = f32
        L.gqo_global_scale.argtypes = [P, P, i32, i64, i32, P, P]
        L.gqo_quantize.argtypes = [P, P, i32, i64, P, i32, i32, i32, u64, u32, f32, P]
        L.gqo_quantize_workers.argtypes = [P, P, i32, i64, P, u32, i32, i32, i32, u64, u32,
                                           f32, P]
        L.gqo_code_value.argtypes = [i32, i32, i32]
        L.gqo_code_value.restype = i32
        L.gqo_uniform_multiplier.argtypes = [i32, f32]
        L.gqo_uniform_multiplier.restype = f32
        L.gqo_packed_row_bytes.argtypes = [i32, i64]
        L.gqo_packed_row_bytes.restype = i64
        L.gqo_pack.argtypes = [P, i32, i64, i32, P]
        L.gqo_unpack.argtypes = [P, i32, i64, i32, P]
        L.gqo_aggregate.argtypes = [P, i32, i64, i32, i32, P]
        L.gqo_decode_mean.argtypes = [P, i64, i32, i32, i32, i32, f32, P]
        L.gqo_error_feedback.argtypes = [P, P, P, i32, i64, i32, i32, i32, f32, P]
        L.gqo_logq_quantize.argtypes = [P, i32, i32, P, f32, u64, u32, P, P]
        L.gqo_logq_quantize_workers.argtypes = [P, i32, i32, P, f32, u64, u32, u32, P, P]
        L.gqo_logq_decode_sum.argtypes = [P, P, i32, i32, P, f32, P]
        L.gqo_logq_map.argtypes = [f32, f32]
        L.gqo_logq_map.restype = f32
        L.gqo_logq_decode_one.argtypes = [i32, f32, f32]
        L.gqo_logq_decode_one.restype = f32
        L.gqo_lowrank_fma.argtypes = [P, P, i64, i64, i32, P]
        L.gqo_lowrank_fma.restype = None
        L.gqo_nat_quantize_workers.argtypes = [P, i32, i64, P, u32, u64, u32, P]
        L.gqo_nat_value.argtypes = [ctypes.c_uint16]
        L.gqo_nat_value.restype = f32
        L.gqo_nat_decode.argtypes = [P, i64, P]
        L.gqo_nat_decode_sum.argtypes = [P, i32, i64, P]
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f32(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float32)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments (rc={rc})")


def philox4x32(ctr, key, rounds=10):
    c = np.ascontiguousarray(np.asarray(ctr, dtype=np.uint32).copy())
    lib().gqo_philox4x32(_p(c), int(key[0]) & 0xFFFFFFFF, int(key[1]) & 0xFFFFFFFF,
                         rounds)
    return c


def uniform_bits(seed, tag, step, worker, j):
    return lib().gqo_uniform_bits(seed, tag, step, worker, j)


def sumsq(g, e=None):
    g = _f32(g)
    e = _f32(e)
    return lib().gqo_sumsq(_p(g), _p(e), g.size)


def sumsq_from(acc, g, e=None):
    """acc + sum of squares of fl(g+e), continuing one ascending fp64 sum."""
    g = _f32(g)
    e = _f32(e)
    return lib().gqo_sumsq_from(float(acc), _p(g), _p(e), g.size)


def maxabs(g, e=None):
    g = _f32(g)
    e = _f32(e)
    return np.float32(lib().gqo_maxabs(_p(g), _p(e), g.size))


def global_scale(g, e=None, scale_kind=SCALE_L2):
    """g, e: [W][d] float32.  Returns (S, norms[W] float64)."""
    g = _f32(g)
    e = _f32(e)
    W, d = g.shape
    S = np.zeros(1, np.float32)
    norms = np.zeros(W, np.float64)
    _check(lib().gqo_global_scale(_p(g), _p(e), W, d, scale_kind, _p(S), _p(norms)),
           "global_scale")
    return np.float32(S[0]), norms


def quantize(g, e=None, *, levels=UNIFORM, s=15, L=8, seed=0, step=0, S, js=None, worker0=0):
    """Codes [W][n] int32 for v = g + e at coordinates js (default 0..n-1); row w
    draws its uniforms as worker worker0 + w."""
    g = _f32(g)
    e = _f32(e)
    W, n = g.shape
    jsa = None if js is None else np.ascontiguousarray(js, dtype=np.int64)
    out = np.zeros((W, n), np.int32)
    _check(lib().gqo_quantize_workers(_p(g), _p(e), W, n, _p(jsa), int(worker0), levels, s, L,
                                      seed, step, float(S), _p(out)), "quantize")
    return out


def uniform_multiplier(s, S):
    return np.float32(lib().gqo_uniform_multiplier(int(s), float(S)))


def code_value(code, levels, L=8):
    return lib().gqo_code_value(int(code), levels, L)


def packed_row_bytes(bits, d):
    return lib().gqo_packed_row_bytes(bits, d)


def pack(codes, bits):
    codes = np.ascontiguousarray(codes, dtype=np.int32)
    W, d = codes.shape
    rb = packed_row_bytes(bits, d)
    if rb < 0:
        raise ValueError("bad bit width")
    out = np.zeros((W, rb), np.uint8)
    _check(lib().gqo_pack(_p(codes), W, d, bits, _p(out)), "pack")
    return out


def unpack(packed, W, d, bits):
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    out = np.zeros((W, d), np.int32)
    _check(lib().gqo_unpack(_p(packed), W, d, bits, _p(out)), "unpack")
    return out


def aggregate(codes, *, levels=UNIFORM, L=8):
    codes = np.ascontiguousarray(codes, dtype=np.int32)
    W, n = codes.shape
    out = np.zeros(n, np.int32)
    _check(lib().gqo_aggregate(_p(codes), W, n, levels, L, _p(out)), "aggregate")
    return out


def decode_mean(sum_, W, *, levels=UNIFORM, s=15, L=8, S):
    sum_ = np.ascontiguousarray(sum_, dtype=np.int32)
    out = np.zeros(sum_.shape[0], np.float32)
    _check(lib().gqo_decode_mean(_p(sum_), sum_.shape[0], W, levels, s, L, float(S),
                                 _p(out)), "decode_mean")
    return out


def error_feedback(g, e, codes, *, levels=UNIFORM, s=15, L=8, S):
    g = _f32(g)
    e = _f32(e)
    codes = np.ascontiguousarray(codes, dtype=np.int32)
    W, n = g.shape
    out = np.zeros((W, n), np.float32)
    _check(lib().gqo_error_feedback(_p(g), _p(e), _p(codes), W, n, levels, s, L,
                                    float(S), _p(out)), "error_feedback")
    return out


def step(g, e=None, *, levels=UNIFORM, s=15, L=8, scale_kind=SCALE_L2, seed=0,
         step=0, ef=False, bits=None, S=None):
    """The whole path on [W][d] inputs: scale, codes, packed bytes, integer sum,
    decoded mean and (ef=True) the new error buffer.  S, when given, replaces
    the computed scale (the GPU's scale, for bit-exact comparison)."""
    g = _f32(g)
    e = _f32(e) if ef else None
    S_ref, norms = global_scale(g, e, scale_kind)
    S_use = S_ref if S is None else np.float32(S)
    codes = quantize(g, e, levels=levels, s=s, L=L, seed=seed, step=step, S=S_use)
    packed = pack(codes, bits) if bits else None
    total = aggregate(codes, levels=levels, L=L)
    out = decode_mean(total, g.shape[0], levels=levels, s=s, L=L, S=S_use)
    e_new = error_feedback(g, e, codes, levels=levels, s=s, L=L, S=S_use) if ef else None
    return dict(S=S_ref, norms=norms, codes=codes, packed=packed, sum=total, out=out,
                e=e_new)


def step_bucketed(g, e=None, *, bucket, levels=UNIFORM, s=15, L=8, scale_kind=SCALE_L2,
                  seed=0, step=0, ef=False, bits=None, S=None):
    """The whole path with one scale per bucket of `bucket` consecutive
    coordinates (the last bucket may be shorter).  Per bucket this is exactly
    the global-scale path of "Quantize Once, Train Fast" (Abstract: global norm
    scaling) restricted to the bucket's coordinates: the scale over the slice,
    then quantization at the slice's own coordinate indices (so the uniforms
    are the same as in the unbucketed path), integer sum, decode and error
    feedback with that bucket's scale.  No new arithmetic: a composition of the
    functions above.  S, when given, is the array of K scales to use."""
    g = _f32(g)
    e = _f32(e) if ef else None
    W, d = g.shape
    K = -(-d // bucket)
    S_ref = np.zeros(K, np.float32)
    codes = np.zeros((W, d), np.int32)
    total = np.zeros(d, np.int32)
    out = np.zeros(d, np.float32)
    e_new = np.zeros((W, d), np.float32) if ef else None
    for k in range(K):
        lo, hi = k * bucket, min(d, (k + 1) * bucket)
        gk = g[:, lo:hi]
        ek = None if e is None else e[:, lo:hi]
        S_ref[k], _ = global_scale(gk, ek, scale_kind)
        Sk = S_ref[k] if S is None else np.float32(S[k])
        ck = quantize(gk, ek, levels=levels, s=s, L=L, seed=seed, step=step, S=Sk,
                      js=np.arange(lo, hi, dtype=np.int64))
        codes[:, lo:hi] = ck
        total[lo:hi] = aggregate(ck, levels=levels, L=L)
        out[lo:hi] = decode_mean(total[lo:hi], W, levels=levels, s=s, L=L, S=Sk)
        if ef:
            e_new[:, lo:hi] = error_feedback(gk, ek, ck, levels=levels, s=s, L=L, S=Sk)
    packed = pack(codes, bits) if bits else None
    return dict(S=S_ref, codes=codes, packed=packed, sum=total, out=out, e=e_new)


def lowrank_fma(P, Q):
    """P (n x r) Q^T (m x r) in float32 with the fma chain of gqo_lowrank_fma."""
    P = _f32(P)
    Q = _f32(Q)
    n, r = P.shape
    m = Q.shape[0]
    out = np.zeros((n, m), np.float32)
    lib().gqo_lowrank_fma(_p(P), _p(Q), n, m, r, _p(out))
    return out


def logq_quantize(x, sizes, *, alpha=10.0, seed=0, step=0, worker0=0):
    """x: [W][sum(sizes)] float32.  Returns (maxabs[W][nmats], codes int8)."""
    x = _f32(x)
    W = x.shape[0]
    sz = np.ascontiguousarray(sizes, dtype=np.int64)
    mx = np.zeros((W, sz.size), np.float32)
    codes = np.zeros(x.shape, np.int8)
    _check(lib().gqo_logq_quantize_workers(_p(x), W, sz.size, _p(sz), alpha, seed, step,
                                           int(worker0), _p(mx), _p(codes)), "logq_quantize")
    return mx, codes


def logq_decode_sum(codes, maxabs, sizes, *, alpha=10.0):
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    maxabs = _f32(maxabs)
    sz = np.ascontiguousarray(sizes, dtype=np.int64)
    out = np.zeros(codes.shape[1], np.float32)
    _check(lib().gqo_logq_decode_sum(_p(codes), _p(maxabs), codes.shape[0], sz.size,
                                     _p(sz), alpha, _p(out)), "logq_decode_sum")
    return out


def logq_map(xn, alpha=10.0):
    return lib().gqo_logq_map(xn, alpha)


def logq_decode_one(k, m, alpha=10.0):
    return lib().gqo_logq_decode_one(k, m, alpha)


# --------------------------------------------------------- natural compression
NAT_TAG = 0x4E410000


def nat_quantize(x, *, seed=0, step=0, worker0=0, js=None):
    """[NC] natural compression of [W][n] float32: uint16 codes (sign bit << 8 |
    biased exponent of the signed power of two, or of the signed zero); row w
    draws its uniforms as worker worker0 + w from the stream tagged NAT_TAG, and
    column i as coordinate js[i] (default i)."""
    x = _f32(x)
    W, n = x.shape
    jsa = None if js is None else np.ascontiguousarray(js, dtype=np.int64)
    out = np.zeros((W, n), np.uint16)
    _check(lib().gqo_nat_quantize_workers(_p(x), W, n, _p(jsa), int(worker0), seed, step,
                                          _p(out)), "nat_quantize")
    return out


def nat_decode(codes):
    """The float value of every code (same shape)."""
    c = np.ascontiguousarray(codes, dtype=np.uint16)
    out = np.zeros(c.shape, np.float32)
    _check(lib().gqo_nat_decode(_p(c), c.size, _p(out)), "nat_decode")
    return out


def nat_decode_sum(codes):
    """fp32 sum over workers (rows) in ascending order, from row 0's value."""
    c = np.ascontiguousarray(codes, dtype=np.uint16)
    W, n = c.shape
    out = np.zeros(n, np.float32)
    _check(lib().gqo_nat_decode_sum(_p(c), W, n, _p(out)), "nat_decode_sum")
    return out

