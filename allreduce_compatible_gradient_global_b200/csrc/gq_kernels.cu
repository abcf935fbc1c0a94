// gq_kernels.cu -- the streaming kernels of the quantization path (sm_100a).
//
//  norm_kernel       step 1: per-worker sum of squares (or max |v|), block
//                    partials in the workspace, combined by the last block.
//  quant_kernel      steps 2-5 in one pass: Philox uniforms in registers,
//                    stochastic rounding, warp packing of the codes, integer
//                    sum over workers in registers, decode, error feedback.
//  aggregate_kernel  step 4 from packed codes (split pipeline).
//  dequant_kernel    step 5 from the sum and packed codes (split pipeline).
//
// Thread mapping of the streaming kernels: a warp owns a 128-coordinate block
// (lane l: coordinates 4l..4l+3, one float4 per worker row, one Philox block
// per worker); warps walk the blocks grid-stride, the grid being a whole
// number of waves of resident blocks.
#include <cfloat>

#include "gq_internal.h"
#include "gq_pdl.cuh"

namespace gq {

// ---------------------------------------------------------------------------
// Loads and stores of 4 consecutive coordinates j0..j0+3 of one row.  VEC: the
// row is 16-byte aligned and d % 4 == 0, so the 4 are all in range or all out.
// Out-of-range coordinates read as 0 (which quantizes to code 0).
// ---------------------------------------------------------------------------
template <bool VEC>
__device__ __forceinline__ float4 load4(const float* row, long long j0, long long d) {
    if (VEC) {
        if (j0 < d) return __ldcs(reinterpret_cast<const float4*>(row + j0));
        return make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float4 r;
    r.x = j0 < d ? __ldcs(row + j0) : 0.f;
    r.y = j0 + 1 < d ? __ldcs(row + j0 + 1) : 0.f;
    r.z = j0 + 2 < d ? __ldcs(row + j0 + 2) : 0.f;
    r.w = j0 + 3 < d ? __ldcs(row + j0 + 3) : 0.f;
    return r;
}

template <bool VEC>
__device__ __forceinline__ void store4(float* row, long long j0, long long d, float4 v) {
    if (VEC || j0 + 3 < d) {
        if (VEC && j0 >= d) return;
        if (VEC) {
            __stcs(reinterpret_cast<float4*>(row + j0), v);
        } else {
            __stcs(row + j0, v.x);
            __stcs(row + j0 + 1, v.y);
            __stcs(row + j0 + 2, v.z);
            __stcs(row + j0 + 3, v.w);
        }
        return;
    }
    if (j0 < d) __stcs(row + j0, v.x);
    if (j0 + 1 < d) __stcs(row + j0 + 1, v.y);
    if (j0 + 2 < d) __stcs(row + j0 + 2, v.z);
}

// Scale-derived constants: a (magnitude multiplier) and c (value of one unit).
template <int LEVELS>
__device__ __forceinline__ void scale_constants(float S, float smax, float finest, float& a,
                                                float& c) {
    const bool ok = S > 0.f && S <= FLT_MAX;
    if (LEVELS == 0) {
        a = ok ? __fdiv_rd(smax, S) : 0.f;  // s/S rounded down: |v| a <= s when |v| <= S
        c = __fdiv_rn(S, smax);
    } else {
        a = ok ? __fdiv_rd(1.0f, S) : 0.f;  // 1/S rounded down: |v| a <= 1 when |v| <= S
        c = __fmul_rn(S, finest);
    }
}

// ---------------------------------------------------------------------------
// Step 1: global scale.
// ---------------------------------------------------------------------------
__device__ __forceinline__ double warp_sum_d(double x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(kFull, x, o);
    return x;
}
__device__ __forceinline__ unsigned warp_max_u(unsigned x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = max(x, __shfl_xor_sync(kFull, x, o));
    return x;
}

// Both kinds track max |v|: it is the scale of the max-abs kind, and for the
// L2 kind it is a floor the rounded norm must not fall below (see the end of
// norm_kernel).  |v| as unsigned bits is order-preserving for non-negative
// floats, and any NaN compares above +Inf, so a NaN input surfaces in the max.
template <int KIND, bool HAS_E>
__device__ __forceinline__ void norm_accum4(float4 x, float4 ex, float& s16, unsigned& mx) {
    if (HAS_E) x = add4(x, ex);
    if (KIND == 0) {
        s16 = __fmaf_rn(x.x, x.x, s16);
        s16 = __fmaf_rn(x.y, x.y, s16);
        s16 = __fmaf_rn(x.z, x.z, s16);
        s16 = __fmaf_rn(x.w, x.w, s16);
    }
    mx = max(mx, __float_as_uint(fabsf(x.x)));
    mx = max(mx, __float_as_uint(fabsf(x.y)));
    mx = max(mx, __float_as_uint(fabsf(x.z)));
    mx = max(mx, __float_as_uint(fabsf(x.w)));
}

// Loads of the norm pass.  Without an error buffer the gradient is read
// evict-first: the pass is bound by DRAM reads, and with its own lines first in
// line for eviction it does not push out (and write back) the dirty lines the
// previous kernel left in L2; measured, that saves ~10 us of the 143 us pass
// that follows the fused pass at 8 x 25.6 M coordinates.  With an error buffer
// (g and e read, e rewritten by the fused pass) the evict-first form measured
// slower, so that instantiation keeps the default L2 policy.
template <bool STREAM, typename T>
__device__ __forceinline__ T ld_norm(const T* p) {
    return STREAM ? __ldcs(p) : __ldcg(p);
}

template <int KIND, bool HAS_E, bool VEC>
__global__ void __launch_bounds__(kThreads, 8) norm_kernel(const __grid_constant__ NormArgs a) {
    // the rows may come from the previous kernel in the stream; the fused pass
    // that follows may be scheduled as soon as every block is running
    pdl_wait();
    pdl_launch_dependents();
    const int w = blockIdx.y;
    const int b = blockIdx.x;
    const float* gw = a.g + (long long)w * a.d;
    const float* ew = HAS_E ? a.e + (long long)w * a.d : nullptr;
    double acc = 0.0;
    unsigned mx = 0u;
    const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);

    if (VEC) {
        const long long n4 = a.d >> 2;
        const float4* g4 = reinterpret_cast<const float4*>(gw);
        const float4* e4 = reinterpret_cast<const float4*>(ew);
        const long long stride = (long long)a.nb * kThreads;
        long long i = (long long)b * kThreads + threadIdx.x;
        for (; i + 3 * stride < n4; i += 4 * stride) {
            float4 x[4], ex[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) x[k] = ld_norm<!HAS_E>(g4 + i + k * stride);
            if (HAS_E) {
#pragma unroll
                for (int k = 0; k < 4; ++k) ex[k] = ld_norm<!HAS_E>(e4 + i + k * stride);
            }
            float s16 = 0.f;
#pragma unroll
            for (int k = 0; k < 4; ++k) norm_accum4<KIND, HAS_E>(x[k], HAS_E ? ex[k] : z4, s16, mx);
            if (KIND == 0) acc += (double)s16;
        }
        for (; i < n4; i += stride) {
            float s16 = 0.f;
            const float4 ev = HAS_E ? ld_norm<!HAS_E>(e4 + i) : z4;
            norm_accum4<KIND, HAS_E>(ld_norm<!HAS_E>(g4 + i), ev, s16, mx);
            if (KIND == 0) acc += (double)s16;
        }
    } else {
        const long long stride = (long long)a.nb * kThreads;
        for (long long i = (long long)b * kThreads + threadIdx.x; i < a.d; i += 4 * stride) {
            float4 x, ex = z4;
            x.x = ld_norm<!HAS_E>(gw + i);
            x.y = i + stride < a.d ? ld_norm<!HAS_E>(gw + i + stride) : 0.f;
            x.z = i + 2 * stride < a.d ? ld_norm<!HAS_E>(gw + i + 2 * stride) : 0.f;
            x.w = i + 3 * stride < a.d ? ld_norm<!HAS_E>(gw + i + 3 * stride) : 0.f;
            if (HAS_E) {
                ex.x = ld_norm<!HAS_E>(ew + i);
                ex.y = i + stride < a.d ? ld_norm<!HAS_E>(ew + i + stride) : 0.f;
                ex.z = i + 2 * stride < a.d ? ld_norm<!HAS_E>(ew + i + 2 * stride) : 0.f;
                ex.w = i + 3 * stride < a.d ? ld_norm<!HAS_E>(ew + i + 3 * stride) : 0.f;
            }
            float s16 = 0.f;
            norm_accum4<KIND, HAS_E>(x, ex, s16, mx);
            if (KIND == 0) acc += (double)s16;
        }
    }

    // Block partial, fixed reduction order.
    __shared__ double red_d[kThreads / 32];
    __shared__ unsigned red_u[kThreads / 32];
    __shared__ bool am_last;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (KIND == 0) {
        acc = warp_sum_d(acc);
        if (lane == 0) red_d[warp] = acc;
    }
    mx = warp_max_u(mx);
    if (lane == 0) red_u[warp] = mx;
    __syncthreads();
    if (threadIdx.x == 0) {
        double t = 0.0;
        unsigned m = 0u;
        if (KIND == 0)
            for (int k = 0; k < kThreads / 32; ++k) t += red_d[k];
        for (int k = 0; k < kThreads / 32; ++k) m = max(m, red_u[k]);
        // two slots per block: the sum of squares, then max |v|
        unsigned long long* slot = a.partials + 2 * ((long long)w * a.nb + b);
        slot[0] = (unsigned long long)__double_as_longlong(t);
        slot[1] = m;
        __threadfence();
        const unsigned total = (unsigned)a.nb * (unsigned)a.W;
        const unsigned ticket = atomicAdd(&a.hdr->counter, 1u);
        am_last = (ticket == total - 1u);
    }
    __syncthreads();
    if (!am_last) return;

    // The last block: combine the partials of every worker (one warp per
    // worker, lanes strided then a fixed xor tree), then the max over workers.
    __threadfence();
    double best = 0.0;
    bool saw_nan = false;
    for (int ww = warp; ww < a.W; ww += kThreads / 32) {
        const unsigned long long* pw = a.partials + 2 * (long long)ww * a.nb;
        unsigned m = 0u;
        double t = 0.0;
        for (int k = lane; k < a.nb; k += 32) {
            if (KIND == 0) t += __longlong_as_double((long long)__ldcg(pw + 2 * k));
            m = max(m, (unsigned)__ldcg(pw + 2 * k + 1));
        }
        m = warp_max_u(m);
        const double mxv = (double)__uint_as_float(m);
        double nrm, cand;
        if (KIND == 0) {
            nrm = sqrt(warp_sum_d(t));
            // In exact arithmetic ||v_w|| >= max|v_w|; the fp32 partial sums
            // can round the norm just below a dominant entry, so the scale
            // never takes a value below max|v|.  Then S >= |v| for every
            // input, which the fused pass relies on to need no clamp.
            cand = nrm != nrm ? nrm : fmax(nrm, mxv);
        } else {
            nrm = mxv;
            cand = mxv;
        }
        if (lane == 0 && a.norms) a.norms[ww] = nrm;
        if (cand != cand || mxv != mxv) saw_nan = true;
        else best = fmax(best, cand);
    }
    __shared__ double wbest[kThreads / 32];
    __shared__ int wnan[kThreads / 32];
    if (lane == 0) {
        wbest[warp] = best;
        wnan[warp] = saw_nan ? 1 : 0;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        double m = 0.0;
        int nan_any = 0;
        for (int k = 0; k < kThreads / 32; ++k) {
            m = fmax(m, wbest[k]);
            nan_any |= wnan[k];
        }
        const float S = nan_any ? __int_as_float(0x7FC00000) : __double2float_rn(m);
        a.scale[0] = S;
        if (!(S <= FLT_MAX)) atomicOr(&a.hdr->flags, kFlagNonfiniteScale);
        a.hdr->counter = 0u;  // ready for the next call (stream order)
    }
}

int norm_resident_blocks(int kind, bool has_e, bool vec) {
    // resident blocks per SM of the instantiation that will run (cached)
    // (atomic: calls from several host threads may race on the first query)
    static int cache[2][2][2] = {};
    int* c = &cache[kind != 0][has_e][vec];
    int n = __atomic_load_n(c, __ATOMIC_ACQUIRE);
    if (n == 0) {
        const void* fn;
        if (kind == 0) {
            fn = has_e ? (vec ? (const void*)norm_kernel<0, true, true> : (const void*)norm_kernel<0, true, false>)
                       : (vec ? (const void*)norm_kernel<0, false, true> : (const void*)norm_kernel<0, false, false>);
        } else {
            fn = has_e ? (vec ? (const void*)norm_kernel<1, true, true> : (const void*)norm_kernel<1, true, false>)
                       : (vec ? (const void*)norm_kernel<1, false, true> : (const void*)norm_kernel<1, false, false>);
        }
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, kThreads, 0) != cudaSuccess || n < 1)
            n = 1;
        __atomic_store_n(c, n, __ATOMIC_RELEASE);
    }
    return n;
}

cudaError_t launch_norm(const NormArgs& a, bool vec, cudaStream_t st) {
    dim3 grid(a.nb, a.W);
    const bool he = a.e != nullptr;
    const bool pdl = pdl_allowed(st);
#define GQ_NORM(K, E, V) \
    return launch_with_pdl(norm_kernel<K, E, V>, grid, dim3(kThreads), 0, st, pdl, a)
    if (a.kind == 0) {
        if (he) { if (vec) GQ_NORM(0, true, true); else GQ_NORM(0, true, false); }
        else    { if (vec) GQ_NORM(0, false, true); else GQ_NORM(0, false, false); }
    } else {
        if (he) { if (vec) GQ_NORM(1, true, true); else GQ_NORM(1, true, false); }
        else    { if (vec) GQ_NORM(1, false, true); else GQ_NORM(1, false, false); }
    }
#undef GQ_NORM
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Steps 2-5 fused.
// ---------------------------------------------------------------------------
// Tuning of the fused pass: worker rows loaded before any is processed,
// resident blocks per SM the register budget is cut for, and whether warps
// walk the 128-coordinate blocks from the end of the rows (the end of the rows
// is what the norm pass left in L2).
#ifndef GQ_WORKER_BATCH
#define GQ_WORKER_BATCH 4
#endif
#ifndef GQ_QUANT_MIN_BLOCKS
#define GQ_QUANT_MIN_BLOCKS 3
#endif
#ifndef GQ_QUANT_REVERSE
#define GQ_QUANT_REVERSE 0
#endif
constexpr int kWorkerBatch = GQ_WORKER_BATCH;

template <int LEVELS>
__device__ __forceinline__ int quantize_one(float v, float aq, const QuantArgs& a, uint32_t word) {
    if (LEVELS == 0) return quant_uniform(v, aq, a.smax, word);
    return quant_exp(v, aq, a.L, a.finest, a.inv_finest, word);
}

template <int LEVELS, int BITS, bool EF, bool VEC>
__global__ void __launch_bounds__(kThreads, GQ_QUANT_MIN_BLOCKS)
    quant_kernel(const __grid_constant__ QuantArgs a) {
    const int lane = threadIdx.x & 31;
    const long long nblk = (a.d + 127) >> 7;
    const long long wid = ((long long)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const long long nwarps = ((long long)gridDim.x * kThreads) >> 5;
    float aq, c;
    scale_constants<LEVELS>(__ldg(a.scale), a.smax, a.finest, aq, c);
    const uint32_t step = a.step_dev ? __ldg(a.step_dev) : a.step;
    Packer<BITS> pk;
    pk.init(lane);

    for (long long it = wid; it < nblk; it += nwarps) {
        const long long blk = GQ_QUANT_REVERSE ? nblk - 1 - it : it;
        if (a.bq_mult) {  // per-bucket scale of this block
            aq = __ldg(a.bq_mult + (blk >> a.bucket_shift));
            c = __ldg(a.bq_unit + (blk >> a.bucket_shift));
        }
        const long long j0 = (blk << 7) + (lane << 2);
        const unsigned long long q = (unsigned long long)(blk << 5) + (unsigned)lane + a.q0;
        int s0 = 0, s1 = 0, s2 = 0, s3 = 0;
        for (int wb = 0; wb < a.W; wb += kWorkerBatch) {
            float4 gv[kWorkerBatch], ev[kWorkerBatch];
#pragma unroll
            for (int i = 0; i < kWorkerBatch; ++i) {
                if (wb + i < a.W) {
                    gv[i] = load4<VEC>(a.g + (long long)(wb + i) * a.d, j0, a.d);
                    if (EF) ev[i] = load4<VEC>(a.e + (long long)(wb + i) * a.d, j0, a.d);
                }
            }
#pragma unroll
            for (int i = 0; i < kWorkerBatch; ++i) {
                if (wb + i < a.W) {
                    const int w = wb + i;
                    const float4 v = EF ? add4(gv[i], ev[i]) : gv[i];
                    const uint4 rnd = philox10(philox_counter(q, step, a.worker0 + (uint32_t)w), a.rk);
                    const int c0 = quantize_one<LEVELS>(v.x, aq, a, rnd.x);
                    const int c1 = quantize_one<LEVELS>(v.y, aq, a, rnd.y);
                    const int c2 = quantize_one<LEVELS>(v.z, aq, a, rnd.z);
                    const int c3 = quantize_one<LEVELS>(v.w, aq, a, rnd.w);
                    const int v0 = code_value<LEVELS>(c0), v1 = code_value<LEVELS>(c1);
                    const int v2 = code_value<LEVELS>(c2), v3 = code_value<LEVELS>(c3);
                    s0 += v0;
                    s1 += v1;
                    s2 += v2;
                    s3 += v3;
                    if (BITS != 0)
                        pk.store(lane, c0, c1, c2, c3,
                                 a.codes + (long long)w * a.row_bytes + blk * (16 * BITS));
                    if (EF && a.update_e) {
                        float4 en;
                        en.x = __fsub_rn(v.x, __fmul_rn(small_int_to_float(v0), c));
                        en.y = __fsub_rn(v.y, __fmul_rn(small_int_to_float(v1), c));
                        en.z = __fsub_rn(v.z, __fmul_rn(small_int_to_float(v2), c));
                        en.w = __fsub_rn(v.w, __fmul_rn(small_int_to_float(v3), c));
                        store4<VEC>(a.e + (long long)w * a.d, j0, a.d, en);
                    }
                }
            }
        }
        if (a.sum) store_sum(a.sum, a.wire, j0, a.d, s0, s1, s2, s3);
        if (a.out) {
            float4 o;
            o.x = decode_mean(s0, c, a.inv_w, a.w_pow2, a.W);
            o.y = decode_mean(s1, c, a.inv_w, a.w_pow2, a.W);
            o.z = decode_mean(s2, c, a.inv_w, a.w_pow2, a.W);
            o.w = decode_mean(s3, c, a.inv_w, a.w_pow2, a.W);
            store_out4(a.out, j0, a.d, o);
        }
    }
}

template <int LEVELS, int BITS>
static void quant_dispatch_ev(const QuantArgs& a, bool ef, bool vec, int grid, cudaStream_t st) {
    if (ef) {
        if (vec) quant_kernel<LEVELS, BITS, true, true><<<grid, kThreads, 0, st>>>(a);
        else quant_kernel<LEVELS, BITS, true, false><<<grid, kThreads, 0, st>>>(a);
    } else {
        if (vec) quant_kernel<LEVELS, BITS, false, true><<<grid, kThreads, 0, st>>>(a);
        else quant_kernel<LEVELS, BITS, false, false><<<grid, kThreads, 0, st>>>(a);
    }
}

template <int LEVELS>
static void quant_dispatch_bits(const QuantArgs& a, int bits, bool ef, bool vec, int grid,
                                cudaStream_t st) {
    switch (bits) {
        case 0: quant_dispatch_ev<LEVELS, 0>(a, ef, vec, grid, st); break;
        case 4: quant_dispatch_ev<LEVELS, 4>(a, ef, vec, grid, st); break;
        case 5: quant_dispatch_ev<LEVELS, 5>(a, ef, vec, grid, st); break;
        case 8: quant_dispatch_ev<LEVELS, 8>(a, ef, vec, grid, st); break;
        default: quant_dispatch_ev<LEVELS, 16>(a, ef, vec, grid, st); break;
    }
}

cudaError_t launch_quant(const QuantArgs& a, int levels, int bits, bool ef, bool vec, int grid,
                         cudaStream_t st) {
    if (levels == 0) quant_dispatch_bits<0>(a, bits, ef, vec, grid, st);
    else quant_dispatch_bits<1>(a, bits, ef, vec, grid, st);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Step 4 from packed codes.
// ---------------------------------------------------------------------------
template <int LEVELS, int BITS>
__global__ void __launch_bounds__(kThreads) aggregate_kernel(const __grid_constant__ AggArgs a) {
    const int lane = threadIdx.x & 31;
    const long long nblk = (a.d + 127) >> 7;
    const long long wid = ((long long)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const long long nwarps = ((long long)gridDim.x * kThreads) >> 5;
    Unpacker<BITS> up;
    up.init(lane);
    for (long long blk = wid; blk < nblk; blk += nwarps) {
        const long long j0 = (blk << 7) + (lane << 2);
        int s0 = 0, s1 = 0, s2 = 0, s3 = 0;
        for (int w = 0; w < a.W; ++w) {
            int c0, c1, c2, c3;
            up.load(lane, a.codes + (long long)w * a.row_bytes + blk * (16 * BITS), c0, c1, c2, c3);
            s0 += code_value<LEVELS>(c0);
            s1 += code_value<LEVELS>(c1);
            s2 += code_value<LEVELS>(c2);
            s3 += code_value<LEVELS>(c3);
        }
        store_sum(a.sum, a.wire, j0, a.d, s0, s1, s2, s3);
    }
}

cudaError_t launch_aggregate(const AggArgs& a, int levels, int bits, int grid, cudaStream_t st) {
#define GQ_AGG(LV, B) aggregate_kernel<LV, B><<<grid, kThreads, 0, st>>>(a)
    if (levels == 0) {
        switch (bits) {
            case 4: GQ_AGG(0, 4); break;
            case 5: GQ_AGG(0, 5); break;
            case 8: GQ_AGG(0, 8); break;
            default: GQ_AGG(0, 16); break;
        }
    } else {
        switch (bits) {
            case 4: GQ_AGG(1, 4); break;
            case 5: GQ_AGG(1, 5); break;
            case 8: GQ_AGG(1, 8); break;
            default: GQ_AGG(1, 16); break;
        }
    }
#undef GQ_AGG
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Step 5 from the sum and the packed codes.
// ---------------------------------------------------------------------------
template <int LEVELS, int BITS, bool VEC>
__global__ void __launch_bounds__(kThreads) dequant_kernel(const __grid_constant__ DequantArgs a) {
    const int lane = threadIdx.x & 31;
    const long long nblk = (a.d + 127) >> 7;
    const long long wid = ((long long)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const long long nwarps = ((long long)gridDim.x * kThreads) >> 5;
    float aq, c;
    scale_constants<LEVELS>(__ldg(a.scale), a.smax, a.finest, aq, c);
    (void)aq;
    Unpacker<BITS> up;
    up.init(lane);
    for (long long blk = wid; blk < nblk; blk += nwarps) {
        const long long j0 = (blk << 7) + (lane << 2);
        if (a.sum) {
            int s0, s1, s2, s3;
            load_sum(a.sum, a.wire, j0, a.d, s0, s1, s2, s3);
            float4 o;
            o.x = decode_mean(s0, c, a.inv_w, a.w_pow2, a.W);
            o.y = decode_mean(s1, c, a.inv_w, a.w_pow2, a.W);
            o.z = decode_mean(s2, c, a.inv_w, a.w_pow2, a.W);
            o.w = decode_mean(s3, c, a.inv_w, a.w_pow2, a.W);
            store_out4(a.out, j0, a.d, o);
        }
        if (a.e) {
            for (int w = 0; w < a.W; ++w) {
                int c0, c1, c2, c3;
                up.load(lane, a.codes + (long long)w * a.row_bytes + blk * (16 * BITS), c0, c1,
                        c2, c3);
                const float4 gv = load4<VEC>(a.g + (long long)w * a.d, j0, a.d);
                const float4 ev = load4<VEC>(a.e + (long long)w * a.d, j0, a.d);
                const float4 v = add4(gv, ev);
                float4 en;
                en.x = __fsub_rn(v.x, __fmul_rn(small_int_to_float(code_value<LEVELS>(c0)), c));
                en.y = __fsub_rn(v.y, __fmul_rn(small_int_to_float(code_value<LEVELS>(c1)), c));
                en.z = __fsub_rn(v.z, __fmul_rn(small_int_to_float(code_value<LEVELS>(c2)), c));
                en.w = __fsub_rn(v.w, __fmul_rn(small_int_to_float(code_value<LEVELS>(c3)), c));
                store4<VEC>(a.e + (long long)w * a.d, j0, a.d, en);
            }
        }
    }
}

cudaError_t launch_dequant(const DequantArgs& a, int levels, int bits, bool vec, int grid,
                           cudaStream_t st) {
#define GQ_DQ(LV, B)                                                          \
    do {                                                                      \
        if (vec) dequant_kernel<LV, B, true><<<grid, kThreads, 0, st>>>(a);   \
        else dequant_kernel<LV, B, false><<<grid, kThreads, 0, st>>>(a);      \
    } while (0)
    if (levels == 0) {
        switch (bits) {
            case 4: GQ_DQ(0, 4); break;
            case 5: GQ_DQ(0, 5); break;
            case 8: GQ_DQ(0, 8); break;
            default: GQ_DQ(0, 16); break;
        }
    } else {
        switch (bits) {
            case 4: GQ_DQ(1, 4); break;
            case 5: GQ_DQ(1, 5); break;
            case 8: GQ_DQ(1, 8); break;
            default: GQ_DQ(1, 16); break;
        }
    }
#undef GQ_DQ
    return cudaGetLastError();
}

// The device step counter of captured step graphs.
__global__ void advance_step_kernel(unsigned int* step_dev, unsigned int by) { *step_dev += by; }

cudaError_t launch_advance_step(unsigned int* step_dev, unsigned int by, cudaStream_t st) {
    advance_step_kernel<<<1, 1, 0, st>>>(step_dev, by);
    return cudaGetLastError();
}

}  // namespace gq
