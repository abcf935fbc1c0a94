// gq_logq.cu -- the LQ-SGD log quantizer on low-rank factors (sm_100a).
//
// "Trustworthy Efficient Communication for Distributed Learning using LQ-SGD
// Algorithm" (review): "Core claim" -- q(x) = sign(x) log(1 + a|x|)/log(1 + a)
// on the entries of the factors P and Q, 2^b uniformly spaced bins, b = 8;
// referee major comment 1 (Section IV-A, Eqs. (5)-(6)) -- the map is bounded
// only after normalising by the maximum magnitude, and Eq. (6) inverts it.
// Bins: sign + 127 magnitude steps of |q| in [0, 1], stochastic rounding.
//
// logq_quantize_kernel: one block per (matrix, worker); pass 1 reduces
// max |x| over the matrix, pass 2 re-reads it (from L2, so DRAM sees one read:
// a factor is at most a few hundred KB) and writes int8 codes.  Where the
// matrix starts on a 16-byte boundary both passes move 16-byte vectors, four
// consecutive entries, which are exactly one Philox block, and the codes
// leave as 4-byte words; otherwise one entry at a time, same arithmetic.
//
// logq_decode_kernel: Eq. (6) and an fp32 sum over workers in ascending
// order.  The inverse map of a magnitude step m, fl(expm1f(fl(fl(m/127) l))/a)
// with l = log1pf(a), does not depend on the worker or the matrix, so each
// block tabulates its values once in shared memory with exactly that
// expression; a code then costs one table read and one multiply by the
// matrix's max, bit for bit what evaluating Eq. (6) per code gives.
#include <cfloat>

#include "gq_internal.h"

namespace gq {

constexpr int kLogqThreads = 512;

// a / b for 0 <= a <= b, given rb = RN(1/b): q0 = RN(a rb) is within an ulp
// of a/b, the remainder r = a - q0 b is exact in one fused multiply-add, and
// RN(q0 + r rb) is the correctly rounded quotient (Markstein, "Computation of
// elementary functions on the IBM RISC System/6000 processor", IBM J. Res.
// Develop. 34(1), 1990) -- provided neither the reciprocal, the remainder nor
// the correction underflows or overflows.  The domain: a divisor in
// [2^-125, 2^125) (a normal, finite reciprocal; fma_div_ok) and a dividend
// that is 0 (exact either way) or at least lo = 2^-100 max(1, b)
// (fma_div_floor); everything else takes IEEE division.  Measured equal to
// IEEE division on 1.7e10 sampled quotients in that domain over 255 divisors
// from 2^-110 to 2^110, edge mantissas and log1p(10) among them; outside it
// the correction alone missed on 0.6% of samples, and for the divisor
// FLT_MAX on 7 in 6.7e7.
__device__ __forceinline__ bool fma_div_ok(float b) { return b >= 0x1p-125f && b < 0x1p125f; }

__device__ __forceinline__ float fma_div_floor(float b) { return 0x1p-100f * fmaxf(1.0f, b); }

__device__ __forceinline__ float div_by_reciprocal(float a, float b, float rb, float lo,
                                                   bool ok) {
    if (!ok || (a < lo && a != 0.f)) return __fdiv_rn(a, b);
    const float q0 = __fmul_rn(a, rb);
    const float r = __fmaf_rn(-q0, b, a);
    return __fmaf_rn(r, rb, q0);
}

__device__ __forceinline__ uint4 philox10_key(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        const unsigned long long p0 = (unsigned long long)c.x * 0xD2511F53ull;
        const unsigned long long p1 = (unsigned long long)c.z * 0xCD9E8D57ull;
        c = make_uint4((uint32_t)(p1 >> 32) ^ c.y ^ k0, (uint32_t)p1,
                       (uint32_t)(p0 >> 32) ^ c.w ^ k1, (uint32_t)p0);
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
    return c;
}

// The corrected quotient without the domain check, for callers that checked it.
__device__ __forceinline__ float div_by_reciprocal_in_domain(float a, float b, float rb) {
    const float q0 = __fmul_rn(a, rb);
    const float r = __fmaf_rn(-q0, b, a);
    return __fmaf_rn(r, rb, q0);
}

// Magnitude step of y = 127 t on the log map, rounded with the uniform of
// `word`, and the sign of v.
__device__ __forceinline__ int logq_round(float tq, float v, uint32_t word) {
    const float y = fminf(__fmul_rn(tq, 127.0f), 127.0f);
    return with_sign_of(floor_y_plus_u(y, unit_plus_u(word)), v);
}

// Whether four non-negative dividends all lie in the corrected quotient's
// domain: each is 0 (exact either way) or at least lo.  On the bit patterns
// minus one, compared unsigned, 0 wraps to the largest value and the order of
// the rest is the order of the floats.
__device__ __forceinline__ bool in_domain4(float a0, float a1, float a2, float a3, float lo) {
    const uint32_t m = min(min(__float_as_uint(a0) - 1u, __float_as_uint(a1) - 1u),
                           min(__float_as_uint(a2) - 1u, __float_as_uint(a3) - 1u));
    return m >= __float_as_uint(lo) - 1u;
}

// Four codes from one Philox block.  Each division takes the corrected
// quotient when all four dividends lie in its domain, IEEE division for all
// four otherwise: the same quotients either way, with one domain check per
// four entries instead of one per entry.
__device__ __forceinline__ uint32_t logq_codes4(float4 v, float M, float alpha, float lam,
                                                float rM, float rlam, float loM, float lolam,
                                                bool okM, bool oklam, uint4 rnd) {
    const float a0 = fabsf(v.x), a1 = fabsf(v.y), a2 = fabsf(v.z), a3 = fabsf(v.w);
    float x0, x1, x2, x3;
    if (okM && in_domain4(a0, a1, a2, a3, loM)) {
        x0 = div_by_reciprocal_in_domain(a0, M, rM);
        x1 = div_by_reciprocal_in_domain(a1, M, rM);
        x2 = div_by_reciprocal_in_domain(a2, M, rM);
        x3 = div_by_reciprocal_in_domain(a3, M, rM);
    } else {
        x0 = __fdiv_rn(a0, M);
        x1 = __fdiv_rn(a1, M);
        x2 = __fdiv_rn(a2, M);
        x3 = __fdiv_rn(a3, M);
    }
    const float l0 = log1pf(__fmul_rn(alpha, x0)), l1 = log1pf(__fmul_rn(alpha, x1));
    const float l2 = log1pf(__fmul_rn(alpha, x2)), l3 = log1pf(__fmul_rn(alpha, x3));
    float t0, t1, t2, t3;
    if (oklam && in_domain4(l0, l1, l2, l3, lolam)) {
        t0 = div_by_reciprocal_in_domain(l0, lam, rlam);
        t1 = div_by_reciprocal_in_domain(l1, lam, rlam);
        t2 = div_by_reciprocal_in_domain(l2, lam, rlam);
        t3 = div_by_reciprocal_in_domain(l3, lam, rlam);
    } else {
        t0 = __fdiv_rn(l0, lam);
        t1 = __fdiv_rn(l1, lam);
        t2 = __fdiv_rn(l2, lam);
        t3 = __fdiv_rn(l3, lam);
    }
    const int c0 = logq_round(t0, v.x, rnd.x), c1 = logq_round(t1, v.y, rnd.y);
    const int c2 = logq_round(t2, v.z, rnd.z), c3 = logq_round(t3, v.w, rnd.w);
    return (uint32_t)(c0 & 255) | ((uint32_t)(c1 & 255) << 8) | ((uint32_t)(c2 & 255) << 16) |
           ((uint32_t)c3 << 24);
}

// One code: the magnitude step of |x| / M on the log map, stochastically
// rounded with the uniform of `word`, and x's sign.  Both divisions of the map
// (by the matrix's max and by log1p(a)) use the divisors' reciprocals rM,
// rlam and floors loM, lolam (div_by_reciprocal).
__device__ __forceinline__ int logq_code(float xv, float M, bool usable, float alpha, float lam,
                                         float rM, float rlam, float loM, float lolam, bool okM,
                                         bool oklam, uint32_t word) {
    int k = 0;
    if (usable) {
        const float xn = div_by_reciprocal(fabsf(xv), M, rM, loM, okM);
        const float lg = log1pf(__fmul_rn(alpha, xn));
        const float tq = div_by_reciprocal(lg, lam, rlam, lolam, oklam);
        const float y = fminf(__fmul_rn(tq, 127.0f), 127.0f);
        k = floor_y_plus_u(y, unit_plus_u(word));
    }
    return with_sign_of(k, xv);
}

// Three 512-thread blocks per SM (40 registers): 384 (worker, matrix) blocks
// of the LQ-SGD workload then run in one wave.
__global__ void __launch_bounds__(kLogqThreads, 3)
    logq_quantize_kernel(const __grid_constant__ LogqArgs a) {
    const int mi = blockIdx.x;  // matrix within this launch
    const int w = blockIdx.y;
    const int m = a.m0 + mi;
    const long long n = a.off[mi + 1] - a.off[mi];
    const long long base = (long long)w * a.total + a.off[mi];
    const float* x = a.x + base;
    signed char* codes = a.codes + base;
    // 16-byte vectors when the matrix's first entry and first code allow them
    const bool vec = ((reinterpret_cast<uintptr_t>(x) & 15u) == 0) &&
                     ((reinterpret_cast<uintptr_t>(codes) & 3u) == 0);
    const long long n4 = vec ? n >> 2 : 0;  // whole 4-entry groups taken as vectors

    unsigned mx0 = 0u, mx1 = 0u;
    {
        const float4* x4 = reinterpret_cast<const float4*>(x);
        long long q = threadIdx.x;
        for (; q + kLogqThreads < n4; q += 2 * kLogqThreads) {  // two vectors in flight
            const float4 u = __ldg(x4 + q), v = __ldg(x4 + q + kLogqThreads);
            mx0 = max(mx0, max(max(__float_as_uint(fabsf(u.x)), __float_as_uint(fabsf(u.y))),
                               max(__float_as_uint(fabsf(u.z)), __float_as_uint(fabsf(u.w)))));
            mx1 = max(mx1, max(max(__float_as_uint(fabsf(v.x)), __float_as_uint(fabsf(v.y))),
                               max(__float_as_uint(fabsf(v.z)), __float_as_uint(fabsf(v.w)))));
        }
        if (q < n4) {
            const float4 u = __ldg(x4 + q);
            mx0 = max(mx0, max(max(__float_as_uint(fabsf(u.x)), __float_as_uint(fabsf(u.y))),
                               max(__float_as_uint(fabsf(u.z)), __float_as_uint(fabsf(u.w)))));
        }
        for (long long i = 4 * n4 + threadIdx.x; i < n; i += kLogqThreads)
            mx1 = max(mx1, __float_as_uint(fabsf(__ldg(x + i))));
    }
    unsigned mx = max(mx0, mx1);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(kFull, mx, o));
    __shared__ unsigned red[kLogqThreads / 32];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
    __syncthreads();
    unsigned all = 0u;
    for (int k = 0; k < kLogqThreads / 32; ++k) all = max(all, red[k]);
    const float M = __uint_as_float(all);
    if (threadIdx.x == 0) {
        a.maxabs[(long long)w * a.nmats + m] = M;
        if (!(M <= FLT_MAX)) atomicOr(&a.hdr->flags, kFlagNonfiniteLogqMax);
    }
    const bool usable = M > 0.f && M <= FLT_MAX;
    const float alpha = a.alpha;
    const float lam = log1pf(alpha);
    const uint32_t k0 = a.seed_lo, k1 = a.seed_hi ^ (0x4C510000u | (uint32_t)m);
    const uint32_t step = a.step_dev ? __ldg(a.step_dev) : a.step;
    const uint32_t wid = a.worker0 + (uint32_t)w;
    const float rM = __frcp_rn(M), rlam = __frcp_rn(lam);
    const float loM = fma_div_floor(M), lolam = fma_div_floor(lam);
    const bool okM = fma_div_ok(M), oklam = fma_div_ok(lam);

    // entries 4q..4q+3 share Philox block q
    const float4* x4 = reinterpret_cast<const float4*>(x);
    for (long long q = threadIdx.x; q < n4; q += kLogqThreads) {
        const float4 v = x4[q];  // an L2 hit: pass 1 just read it
        const uint4 rnd =
            philox10_key(philox_counter((unsigned long long)q, step, wid), k0, k1);
        reinterpret_cast<uint32_t*>(codes)[q] =
            usable ? logq_codes4(v, M, alpha, lam, rM, rlam, loM, lolam, okM, oklam, rnd) : 0u;
    }
    // the rest one entry at a time (all of it when the matrix is not aligned)
    for (long long q = n4 + threadIdx.x; 4 * q < n; q += kLogqThreads) {
        const uint4 rnd =
            philox10_key(philox_counter((unsigned long long)q, step, wid), k0, k1);
        const uint32_t words[4] = {rnd.x, rnd.y, rnd.z, rnd.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const long long i = 4 * q + t;
            if (i < n)
                codes[i] = (signed char)logq_code(__ldg(x + i), M, usable, alpha, lam, rM,
                                                  rlam, loM, lolam, okM, oklam, words[t]);
        }
    }
}

// The inverse map of magnitude step m (Eq. (6) without the max), m = 0..128
// (128 only from a caller's code -128, which the quantizer never writes).
__device__ __forceinline__ float logq_unit_value(int m, float alpha, float lam) {
    const float z = __fmul_rn(__fdiv_rn((float)m, 127.0f), lam);
    return __fdiv_rn(expm1f(z), alpha);
}

__device__ __forceinline__ float logq_decode_one(int k, float M, const float* tab) {
    const float xm = __fmul_rn(tab[k < 0 ? -k : k], M);
    return k < 0 ? -xm : xm;
}

__global__ void __launch_bounds__(kLogqThreads)
    logq_decode_kernel(const __grid_constant__ LogqArgs a) {
    __shared__ float tab[129];  // every int8 magnitude, 0..128
    const float alpha = a.alpha;
    const float lam = log1pf(alpha);
    if (threadIdx.x < 129) tab[threadIdx.x] = logq_unit_value((int)threadIdx.x, alpha, lam);
    __syncthreads();
    const int mi = blockIdx.y;
    const int m = a.m0 + mi;
    const long long n = a.off[mi + 1] - a.off[mi];
    const long long off = a.off[mi];
    // 4-byte code words and 16-byte outputs when every row's slice allows them
    const bool vec = ((off & 3) == 0) && ((a.total & 3) == 0) &&
                     ((reinterpret_cast<uintptr_t>(a.ccodes) & 3u) == 0) &&
                     ((reinterpret_cast<uintptr_t>(a.out) & 15u) == 0);
    const long long n4 = vec ? n >> 2 : 0;
    const long long stride = (long long)gridDim.x * kLogqThreads;
    for (long long q = (long long)blockIdx.x * kLogqThreads + threadIdx.x; q < n4; q += stride) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int w = 0; w < a.W; ++w) {
            const uint32_t c = __ldcs(reinterpret_cast<const unsigned int*>(
                a.ccodes + (long long)w * a.total + off) + q);
            const float M = __ldg(a.cmaxabs + (long long)w * a.nmats + m);
            acc.x = __fadd_rn(acc.x, logq_decode_one((int)(signed char)(c & 255), M, tab));
            acc.y = __fadd_rn(acc.y, logq_decode_one((int)(signed char)((c >> 8) & 255), M, tab));
            acc.z = __fadd_rn(acc.z, logq_decode_one((int)(signed char)((c >> 16) & 255), M, tab));
            acc.w = __fadd_rn(acc.w, logq_decode_one((int)(signed char)(c >> 24), M, tab));
        }
        __stcs(reinterpret_cast<float4*>(a.out + off) + q, acc);
    }
    for (long long i = 4 * n4 + (long long)blockIdx.x * kLogqThreads + threadIdx.x; i < n;
         i += stride) {
        float acc = 0.f;
        for (int w = 0; w < a.W; ++w) {
            const int k = a.ccodes[(long long)w * a.total + off + i];
            const float M = __ldg(a.cmaxabs + (long long)w * a.nmats + m);
            acc = __fadd_rn(acc, logq_decode_one(k, M, tab));
        }
        a.out[off + i] = acc;
    }
}

// Self-test of the log map's division: out[i] = a[i] / b as the quantize
// kernel computes it (div_by_reciprocal with b's reciprocal and floor).
__global__ void fma_div_selftest_kernel(const float* a, float b, float* out, long long n) {
    const float rb = __frcp_rn(b), lo = fma_div_floor(b);
    const bool ok = fma_div_ok(b);
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (long long)gridDim.x * blockDim.x)
        out[i] = div_by_reciprocal(a[i], b, rb, lo, ok);
}

cudaError_t launch_fma_div_selftest(const float* a, float b, float* out, long long n, int sms,
                                    cudaStream_t st) {
    long long blocks = (n + 255) / 256;
    if (blocks > (long long)sms * 8) blocks = (long long)sms * 8;
    if (blocks < 1) blocks = 1;
    fma_div_selftest_kernel<<<(unsigned)blocks, 256, 0, st>>>(a, b, out, n);
    return cudaGetLastError();
}

cudaError_t launch_logq_quantize(const LogqArgs& a, cudaStream_t st) {
    dim3 grid(a.count, a.W);
    logq_quantize_kernel<<<grid, kLogqThreads, 0, st>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_logq_decode(const LogqArgs& a, cudaStream_t st) {
    long long maxn = 0;
    for (int i = 0; i < a.count; ++i) maxn = max(maxn, a.off[i + 1] - a.off[i]);
    // a thread takes 4 coordinates where the vectors apply, 1 elsewhere (two
    // groups per thread, so that the grid fits one wave, measured slower:
    // 16.4 against 13.3 us at rank 7)
    long long bx = (maxn / 4 + kLogqThreads - 1) / kLogqThreads;
    if (bx < 1) bx = 1;
    if (bx > 64) bx = 64;
    dim3 grid((unsigned)bx, a.count);
    logq_decode_kernel<<<grid, kLogqThreads, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace gq
