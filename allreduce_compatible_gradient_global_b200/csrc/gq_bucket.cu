// gq_bucket.cu -- per-bucket global scales (sm_100a).
//
// The global scale of "Quantize Once, Train Fast: Allreduce-Compatible
// Compression with Provable Guarantees" (Abstract: global norm scaling) taken
// per bucket of 2^b consecutive coordinates: S_k = max over workers of the
// worker's norm over bucket k (L2 with the same max-abs floor as the global
// scale, or max-abs).  Every worker quantizes bucket k on the same grid, so the
// integer codes of a bucket still sum across workers; a real exchange adds one
// MAX all-reduce of the K scales.
//
// Buckets of at most 2^12 coordinates take one launch:
//   bucket_small_kernel: one block per bucket; each warp reduces whole worker
//     rows of the bucket with shuffles, the block takes the max over workers.
// Larger buckets take two, so that the grid stays one full wave even when
// there are only a few buckets:
//   bucket_partial_kernel: one block per (worker, chunk of 4096 coordinates),
//     grid-stride over all W * nchunks items; each writes the chunk's sum of
//     squares and max |v| bits.
//   bucket_combine_kernel: one block per bucket combines its chunks per worker
//     in a fixed order and takes the max over workers.
// Both write S_k together with the multiplier a_k (s/S_k or 1/S_k, rounded
// down) and the unit c_k that the fused pass reads per 128-coordinate block.
// Sums of squares everywhere: fp32 squares, fp32 runs of at most 16 terms,
// fp64 accumulation, fixed order (so S_k is the same on every run).
#include <cfloat>

#include "gq_internal.h"

namespace gq {

constexpr int kBucketThreads = 256;
constexpr int kSmallBucketLog2Max = 12;  // up to here one launch, a warp per (bucket, worker)

__device__ __forceinline__ double block_sum_d(double x, double* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(kFull, x, o);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    __syncthreads();
    if (lane == 0) red[warp] = x;
    __syncthreads();
    double t = 0.0;
    for (int k = 0; k < kBucketThreads / 32; ++k) t += red[k];
    return t;
}

__device__ __forceinline__ unsigned block_max_u(unsigned x, unsigned* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = max(x, __shfl_xor_sync(kFull, x, o));
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    __syncthreads();
    if (lane == 0) red[warp] = x;
    __syncthreads();
    unsigned t = 0u;
    for (int k = 0; k < kBucketThreads / 32; ++k) t = max(t, red[k]);
    return t;
}

__device__ __forceinline__ void accumulate4(float4 v, float& s, unsigned& mx, bool sq) {
    if (sq) {
        s = __fmaf_rn(v.x, v.x, s);
        s = __fmaf_rn(v.y, v.y, s);
        s = __fmaf_rn(v.z, v.z, s);
        s = __fmaf_rn(v.w, v.w, s);
    }
    mx = max(mx, __float_as_uint(fabsf(v.x)));
    mx = max(mx, __float_as_uint(fabsf(v.y)));
    mx = max(mx, __float_as_uint(fabsf(v.z)));
    mx = max(mx, __float_as_uint(fabsf(v.w)));
}

// Loads of the scale pass, with the same policy as the global norm pass:
// without an error buffer the gradient is read evict-first, so that the pass's
// own lines leave L2 before the dirty lines the previous fused pass left there
// (measured at 8 x 25.6 M coordinates: the bucketed step 363 -> 354-360 us).
template <bool STREAM, typename T>
__device__ __forceinline__ T ld_bucket(const T* p) {
    return STREAM ? __ldcs(p) : __ldcg(p);
}

// VEC: d % 4 == 0 (every row and chunk starts on a 16-byte boundary).
template <int KIND, bool HAS_E, bool VEC>
__global__ void __launch_bounds__(kBucketThreads)
    bucket_partial_kernel(const __grid_constant__ BucketArgs a) {
    __shared__ double red_d[kBucketThreads / 32];
    __shared__ unsigned red_u[kBucketThreads / 32];
    const long long chunk = 1LL << a.chunk_log2;
    const long long items = (long long)a.W * a.nchunks;
    for (long long it = blockIdx.x; it < items; it += gridDim.x) {
        const int w = (int)(it / a.nchunks);
        const long long ci = it - (long long)w * a.nchunks;
        const long long j0 = ci << a.chunk_log2;
        const long long n = a.d - j0 < chunk ? a.d - j0 : chunk;
        const float* gw = a.g + (long long)w * a.d + j0;
        const float* ew = HAS_E ? a.e + (long long)w * a.d + j0 : nullptr;
        double acc = 0.0;
        unsigned mx = 0u;
        if (VEC) {
            const float4* g4 = reinterpret_cast<const float4*>(gw);
            const float4* e4 = reinterpret_cast<const float4*>(ew);
            const long long n4 = n >> 2;
            for (long long i = threadIdx.x; i < n4; i += 4LL * kBucketThreads) {
                float s16 = 0.f;  // a run of at most 16 squares in fp32
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const long long idx = i + (long long)u * kBucketThreads;
                    if (idx < n4) {
                        float4 v = ld_bucket<!HAS_E>(g4 + idx);
                        if (HAS_E) {
                            const float4 ev = ld_bucket<!HAS_E>(e4 + idx);
                            v = make_float4(__fadd_rn(v.x, ev.x), __fadd_rn(v.y, ev.y),
                                            __fadd_rn(v.z, ev.z), __fadd_rn(v.w, ev.w));
                        }
                        accumulate4(v, s16, mx, KIND == 0);
                    }
                }
                if (KIND == 0) acc += (double)s16;
            }
        } else {
            for (long long i = threadIdx.x; i < n; i += 16LL * kBucketThreads) {
                float s16 = 0.f;
#pragma unroll 4
                for (int u = 0; u < 16; ++u) {
                    const long long idx = i + (long long)u * kBucketThreads;
                    if (idx < n) {
                        float v = ld_bucket<!HAS_E>(gw + idx);
                        if (HAS_E) v = __fadd_rn(v, ld_bucket<!HAS_E>(ew + idx));
                        if (KIND == 0) s16 = __fmaf_rn(v, v, s16);
                        mx = max(mx, __float_as_uint(fabsf(v)));
                    }
                }
                if (KIND == 0) acc += (double)s16;
            }
        }
        const unsigned m_all = block_max_u(mx, red_u);
        const double s_all = KIND == 0 ? block_sum_d(acc, red_d) : 0.0;
        if (threadIdx.x == 0) {
            a.part_sum[it] = s_all;
            a.part_max[it] = m_all;
        }
    }
}

// Writes S_k and the table entries from the max over workers (NaN if any
// worker's norm was NaN).
__device__ __forceinline__ void write_bucket(const BucketArgs& a, long long k, double best,
                                             bool saw_nan) {
    const float S = saw_nan ? __int_as_float(0x7FC00000) : __double2float_rn(best);
    const bool ok = S > 0.f && S <= FLT_MAX;
    a.scales[k] = S;
    if (a.levels == 0) {
        a.mult[k] = ok ? __fdiv_rd(a.smax, S) : 0.f;  // |v| a_k <= s for |v| <= S_k
        a.unit[k] = __fdiv_rn(S, a.smax);
    } else {
        a.mult[k] = ok ? __fdiv_rd(1.0f, S) : 0.f;  // |v| a_k <= 1 for |v| <= S_k
        a.unit[k] = __fmul_rn(S, a.finest);
    }
    if (!(S <= FLT_MAX)) atomicOr(&a.hdr->flags, kFlagNonfiniteScale);
}

// One block per bucket; the chunks of a bucket are combined per worker by a
// fixed thread mapping and reduction tree, so S_k is the same on every run.
template <int KIND>
__global__ void __launch_bounds__(kBucketThreads)
    bucket_combine_kernel(const __grid_constant__ BucketArgs a) {
    __shared__ double red_d[kBucketThreads / 32];
    __shared__ unsigned red_u[kBucketThreads / 32];
    const long long per = 1LL << (a.bucket_log2 - a.chunk_log2);  // chunks per bucket
    for (long long k = blockIdx.x; k < a.nbuckets; k += gridDim.x) {
        const long long c0 = k * per;
        const long long c1 = c0 + per < a.nchunks ? c0 + per : a.nchunks;
        double best = 0.0;
        bool saw_nan = false;
        for (int w = 0; w < a.W; ++w) {
            const long long base = (long long)w * a.nchunks;
            double acc = 0.0;
            unsigned mx = 0u;
            for (long long c = c0 + threadIdx.x; c < c1; c += kBucketThreads) {
                if (KIND == 0) acc += a.part_sum[base + c];
                mx = max(mx, a.part_max[base + c]);
            }
            const unsigned m_all = block_max_u(mx, red_u);
            // max |v| as a float (a NaN's bits compare above +inf's)
            const double mxv = (double)__uint_as_float(m_all);
            double cand;
            if (KIND == 0) {
                const double nrm = sqrt(block_sum_d(acc, red_d));
                cand = nrm != nrm ? nrm : fmax(nrm, mxv);  // never below max |v| (rounding repair)
            } else {
                cand = mxv;
            }
            if (cand != cand) saw_nan = true;
            else best = fmax(best, cand);
        }
        if (threadIdx.x == 0) write_bucket(a, k, best, saw_nan);
    }
}

// Buckets of at most 4096 coordinates in one launch: one block per bucket
// (grid-stride); warp i reduces workers i, i + 8, ... over the whole bucket
// with shuffles only (lane-strided fp32 runs of 16 terms, fp64 accumulation,
// a fixed shuffle tree), and the block takes the max over its warps.
template <int KIND, bool HAS_E, bool VEC>
__global__ void __launch_bounds__(kBucketThreads)
    bucket_small_kernel(const __grid_constant__ BucketArgs a) {
    constexpr int kWarps = kBucketThreads / 32;
    __shared__ double best_w[kWarps];
    __shared__ int nan_w[kWarps];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const long long bsize = 1LL << a.bucket_log2;
    for (long long k = blockIdx.x; k < a.nbuckets; k += gridDim.x) {
        const long long j0 = k * bsize;
        const long long n = a.d - j0 < bsize ? a.d - j0 : bsize;
        double best = 0.0;
        bool saw_nan = false;
        for (int w = warp; w < a.W; w += kWarps) {
            const float* gw = a.g + (long long)w * a.d + j0;
            const float* ew = HAS_E ? a.e + (long long)w * a.d + j0 : nullptr;
            double acc = 0.0;
            unsigned mx = 0u;
            if (VEC) {
                const float4* g4 = reinterpret_cast<const float4*>(gw);
                const float4* e4 = reinterpret_cast<const float4*>(ew);
                const int n4 = (int)(n >> 2);
                for (int i = lane; i < n4; i += 4 * 32) {
                    float s16 = 0.f;
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int idx = i + u * 32;
                        if (idx < n4) {
                            float4 v = ld_bucket<!HAS_E>(g4 + idx);
                            if (HAS_E) {
                                const float4 ev = ld_bucket<!HAS_E>(e4 + idx);
                                v = make_float4(__fadd_rn(v.x, ev.x), __fadd_rn(v.y, ev.y),
                                                __fadd_rn(v.z, ev.z), __fadd_rn(v.w, ev.w));
                            }
                            accumulate4(v, s16, mx, KIND == 0);
                        }
                    }
                    if (KIND == 0) acc += (double)s16;
                }
            } else {
                for (int i = lane; i < (int)n; i += 16 * 32) {
                    float s16 = 0.f;
#pragma unroll 4
                    for (int u = 0; u < 16; ++u) {
                        const int idx = i + u * 32;
                        if (idx < (int)n) {
                            float v = ld_bucket<!HAS_E>(gw + idx);
                            if (HAS_E) v = __fadd_rn(v, ld_bucket<!HAS_E>(ew + idx));
                            if (KIND == 0) s16 = __fmaf_rn(v, v, s16);
                            mx = max(mx, __float_as_uint(fabsf(v)));
                        }
                    }
                    if (KIND == 0) acc += (double)s16;
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                mx = max(mx, __shfl_xor_sync(kFull, mx, o));
                if (KIND == 0) acc += __shfl_xor_sync(kFull, acc, o);
            }
            const double mxv = (double)__uint_as_float(mx);
            double cand;
            if (KIND == 0) {
                const double nrm = sqrt(acc);
                cand = nrm != nrm ? nrm : fmax(nrm, mxv);  // never below max |v|
            } else {
                cand = mxv;
            }
            if (cand != cand) saw_nan = true;
            else best = fmax(best, cand);
        }
        if (lane == 0) {
            best_w[warp] = best;
            nan_w[warp] = saw_nan ? 1 : 0;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            double b = 0.0;
            bool nn = false;
            for (int i = 0; i < kWarps; ++i) {
                b = fmax(b, best_w[i]);
                nn = nn || nan_w[i] != 0;
            }
            write_bucket(a, k, b, nn);
        }
        __syncthreads();
    }
}

template <int KIND, bool HAS_E, bool VEC>
const void* partial_fn() {
    return (const void*)bucket_partial_kernel<KIND, HAS_E, VEC>;
}

template <int KIND, bool HAS_E, bool VEC>
const void* small_fn() {
    return (const void*)bucket_small_kernel<KIND, HAS_E, VEC>;
}

static const void* pick(const BucketArgs& a, bool small) {
    const bool he = a.e != nullptr;
    const bool vec = (a.d % 4) == 0;
    if (small) {
        if (a.kind == 0)
            return he ? (vec ? small_fn<0, true, true>() : small_fn<0, true, false>())
                      : (vec ? small_fn<0, false, true>() : small_fn<0, false, false>());
        return he ? (vec ? small_fn<1, true, true>() : small_fn<1, true, false>())
                  : (vec ? small_fn<1, false, true>() : small_fn<1, false, false>());
    }
    if (a.kind == 0)
        return he ? (vec ? partial_fn<0, true, true>() : partial_fn<0, true, false>())
                  : (vec ? partial_fn<0, false, true>() : partial_fn<0, false, false>());
    return he ? (vec ? partial_fn<1, true, true>() : partial_fn<1, true, false>())
              : (vec ? partial_fn<1, false, true>() : partial_fn<1, false, false>());
}

cudaError_t launch_bucket_scales(const BucketArgs& a, int sms, cudaStream_t st) {
    const bool small = a.bucket_log2 <= kSmallBucketLog2Max;
    const void* fn = pick(a, small);
    int per_sm = 0;
    cudaError_t err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kBucketThreads, 0);
    if (err != cudaSuccess) return err;
    if (per_sm < 1) per_sm = 1;
    void* args[] = {const_cast<BucketArgs*>(&a)};
    if (small) {
        const long long cap = (long long)sms * per_sm;
        const int g = (int)(a.nbuckets < cap ? a.nbuckets : cap);
        err = cudaLaunchKernel(fn, dim3(g), dim3(kBucketThreads), args, 0, st);
        return err != cudaSuccess ? err : cudaGetLastError();
    }
    const long long items = (long long)a.W * a.nchunks;
    const long long cap = (long long)sms * per_sm;
    const int g1 = (int)(items < cap ? items : cap);
    err = cudaLaunchKernel(fn, dim3(g1), dim3(kBucketThreads), args, 0, st);
    if (err != cudaSuccess) return err;
    const long long cap2 = (long long)sms * 8;
    const int g2 = (int)(a.nbuckets < cap2 ? a.nbuckets : cap2);
    if (a.kind == 0) bucket_combine_kernel<0><<<g2, kBucketThreads, 0, st>>>(a);
    else bucket_combine_kernel<1><<<g2, kBucketThreads, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace gq
