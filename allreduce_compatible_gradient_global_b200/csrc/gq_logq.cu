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
// max |x| over the matrix, pass 2 re-reads it (from L2: a factor is at most a
// few hundred KB) and writes int8 codes.  logq_decode_kernel: Eq. (6) per
// code and an fp32 sum over workers in ascending order.
#include <cfloat>

#include "gq_internal.h"

namespace gq {

constexpr int kLogqThreads = 512;

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

__global__ void __launch_bounds__(kLogqThreads) logq_quantize_kernel(const __grid_constant__ LogqArgs a) {
    const int mi = blockIdx.x;  // matrix within this launch
    const int w = blockIdx.y;
    const int m = a.m0 + mi;
    const long long n = a.off[mi + 1] - a.off[mi];
    const long long base = (long long)w * a.total + a.off[mi];
    const float* x = a.x + base;
    signed char* codes = a.codes + base;

    unsigned mx = 0u;
    for (long long i = threadIdx.x; i < n; i += kLogqThreads)
        mx = max(mx, __float_as_uint(fabsf(__ldg(x + i))));
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

    // four consecutive entries per thread share one Philox block
    for (long long q = threadIdx.x; 4 * q < n; q += kLogqThreads) {
        const uint4 rnd = philox10_key(philox_counter((unsigned long long)q, step, a.worker0 + (uint32_t)w), k0, k1);
        const uint32_t words[4] = {rnd.x, rnd.y, rnd.z, rnd.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const long long i = 4 * q + t;
            if (i < n) {
                const float xv = __ldg(x + i);
                int k = 0;
                if (usable) {
                    const float xn = __fdiv_rn(fabsf(xv), M);
                    const float tq = __fdiv_rn(log1pf(__fmul_rn(alpha, xn)), lam);
                    const float y = fminf(__fmul_rn(tq, 127.0f), 127.0f);
                    k = floor_y_plus_u(y, unit_plus_u(words[t]));
                }
                codes[i] = (signed char)with_sign_of(k, xv);
            }
        }
    }
}

__global__ void __launch_bounds__(kLogqThreads) logq_decode_kernel(const __grid_constant__ LogqArgs a) {
    const int mi = blockIdx.y;
    const int m = a.m0 + mi;
    const long long n = a.off[mi + 1] - a.off[mi];
    const float alpha = a.alpha;
    const float lam = log1pf(alpha);
    for (long long i = (long long)blockIdx.x * kLogqThreads + threadIdx.x; i < n;
         i += (long long)gridDim.x * kLogqThreads) {
        float acc = 0.f;
        for (int w = 0; w < a.W; ++w) {
            const int k = a.ccodes[(long long)w * a.total + a.off[mi] + i];
            const float M = __ldg(a.cmaxabs + (long long)w * a.nmats + m);
            const int mag = k < 0 ? -k : k;
            const float z = __fmul_rn(__fdiv_rn((float)mag, 127.0f), lam);
            const float xm = __fmul_rn(__fdiv_rn(expm1f(z), alpha), M);
            acc = __fadd_rn(acc, k < 0 ? -xm : xm);
        }
        a.out[a.off[mi] + i] = acc;
    }
}

cudaError_t launch_logq_quantize(const LogqArgs& a, cudaStream_t st) {
    dim3 grid(a.count, a.W);
    logq_quantize_kernel<<<grid, kLogqThreads, 0, st>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_logq_decode(const LogqArgs& a, cudaStream_t st) {
    long long maxn = 0;
    for (int i = 0; i < a.count; ++i) maxn = max(maxn, a.off[i + 1] - a.off[i]);
    long long bx = (maxn + kLogqThreads - 1) / kLogqThreads;
    if (bx < 1) bx = 1;
    if (bx > 64) bx = 64;
    dim3 grid((unsigned)bx, a.count);
    logq_decode_kernel<<<grid, kLogqThreads, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace gq
