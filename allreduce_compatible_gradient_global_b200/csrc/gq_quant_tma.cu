// gq_quant_tma.cu -- the fused second pass (steps 2-5) with the worker rows
// staged in shared memory by bulk asynchronous copies (sm_100a).
//
// Why: the pass is bound by how many bytes are in flight while the SM spends
// ~20 instructions per element on Philox, rounding and packing.  Holding the
// in-flight rows in registers (one float4 per worker per lane) caps the
// resident warps; here a producer warp streams each worker's row segment of
// a 1024-coordinate tile with one cp.async.bulk into a ring of STAGES tiles,
// and eight compute warps read their 128-coordinate block of every row from
// shared memory.  The copies run ahead by STAGES - 1 tiles regardless of how
// long the compute takes.
//
// Synchronization: per stage a "full" mbarrier (one producer arrival plus the
// transaction bytes of the copies) and an "empty" mbarrier (one arrival per
// compute warp).  Every wait is bounded by the global timer; on expiry the
// waiting warp raises a flag in the workspace and leaves its loop, and the
// producer drains the copies it issued before the block exits.
//
// Arithmetic, packing and outputs are those of quant_kernel, bit for bit.
#include <cfloat>

#include "gq_internal.h"

namespace gq {

constexpr int kTmaTile = 1024;  // coordinates per worker row per stage
constexpr int kTmaComputeWarps = kTmaTile / 128;
constexpr int kTmaThreads = (kTmaComputeWarps + 1) * 32;
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for the phase with the given parity to complete, for at most
// kWaitLimitNs; false (and the flag raised) if it never did.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, WsHeader* hdr) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_ns() - t0 > kWaitLimitNs) {
            atomicOr(&hdr->flags, kFlagPipelineTimeout);
            return false;
        }
    }
    return true;
}

// One bulk copy global -> shared (no multicast), completing on `bar`.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(dst), "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

template <int LEVELS>
__device__ __forceinline__ int quantize_tma(float v, float aq, const QuantArgs& a, uint32_t word) {
    if (LEVELS == 0) return quant_uniform(v, aq, a.smax, word);
    return quant_exp(v, aq, a.L, a.finest, a.inv_finest, word);
}

template <int LEVELS, int BITS, bool EF, int STAGES>
__global__ void __launch_bounds__(kTmaThreads, 1)
    quant_tma_kernel(const __grid_constant__ QuantArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    const int rows = EF ? 2 * a.W : a.W;  // g rows, then e rows
    float* buf = reinterpret_cast<float*>(smem);
    unsigned long long* bars = reinterpret_cast<unsigned long long*>(
        smem + (size_t)STAGES * rows * kTmaTile * sizeof(float));
    const uint32_t full0 = smem_addr(bars);
    const uint32_t empty0 = smem_addr(bars + STAGES);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long ntiles = (a.d + kTmaTile - 1) / kTmaTile;
    const long long nblk = (a.d + 127) >> 7;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, kTmaComputeWarps);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    if (warp == kTmaComputeWarps) {
        // ---------------- producer: one lane issues every copy ----------------
        if (lane == 0) {
            long long issued = 0;  // tiles whose copies were issued
            bool ok = true;
            for (long long t = blockIdx.x; t < ntiles; t += gridDim.x, ++issued) {
                const int s = (int)(issued % STAGES);
                if (issued >= STAGES) {
                    const uint32_t par = (uint32_t)((issued / STAGES - 1) & 1);
                    if (!mbar_wait_bounded(empty0 + 8 * s, par, a.hdr)) {
                        ok = false;
                        break;
                    }
                }
                const long long j0 = t * kTmaTile;
                const long long n = a.d - j0 < kTmaTile ? a.d - j0 : kTmaTile;
                const uint32_t bytes = (uint32_t)(n * sizeof(float));
                mbar_arrive_expect_tx(full0 + 8 * s, bytes * (uint32_t)rows);
                for (int r = 0; r < rows; ++r) {
                    const float* src = (r < a.W ? a.g + (long long)r * a.d
                                                : a.e + (long long)(r - a.W) * a.d) + j0;
                    bulk_g2s(smem_addr(buf + ((size_t)s * rows + r) * kTmaTile), src, bytes,
                             full0 + 8 * s);
                }
            }
            // Drain: every issued stage must have landed before the block exits.
            // On the normal path the consumers already waited for all of them;
            // after a timeout, wait (bounded) for the last STAGES issued tiles.
            if (!ok) {
                const long long first = issued > STAGES ? issued - STAGES : 0;
                for (long long k = first; k < issued; ++k)
                    mbar_wait_bounded(full0 + 8 * (int)(k % STAGES), (uint32_t)((k / STAGES) & 1),
                                      a.hdr);
            }
        }
        return;
    }

    // ---------------- compute warps ----------------
    float aq, c;
    {
        const float S = __ldg(a.scale);
        const bool okS = S > 0.f && S <= FLT_MAX;
        if (LEVELS == 0) {
            aq = okS ? __fdiv_rn(a.smax, S) : 0.f;
            c = __fdiv_rn(S, a.smax);
        } else {
            aq = okS ? __fdiv_rn(1.0f, S) : 0.f;
            c = __fmul_rn(S, a.finest);
        }
    }
    Packer<BITS> pk;
    pk.init(lane);
    long long k = 0;
    for (long long t = blockIdx.x; t < ntiles; t += gridDim.x, ++k) {
        const int s = (int)(k % STAGES);
        if (!mbar_wait_bounded(full0 + 8 * s, (uint32_t)((k / STAGES) & 1), a.hdr)) break;
        const long long blk = t * kTmaComputeWarps + warp;
        if (blk < nblk) {
            const long long j0 = (blk << 7) + (lane << 2);
            const bool in = j0 < a.d;  // d % 4 == 0: all four or none
            const unsigned long long q = (unsigned long long)(blk << 5) + (unsigned)lane;
            const float* stage = buf + (size_t)s * rows * kTmaTile + warp * 128 + lane * 4;
            int s0 = 0, s1 = 0, s2 = 0, s3 = 0;
#pragma unroll 2
            for (int w = 0; w < a.W; ++w) {
                float4 v = in ? *reinterpret_cast<const float4*>(stage + (size_t)w * kTmaTile)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
                if (EF && in) {
                    const float4 ev =
                        *reinterpret_cast<const float4*>(stage + (size_t)(a.W + w) * kTmaTile);
                    v = make_float4(__fadd_rn(v.x, ev.x), __fadd_rn(v.y, ev.y),
                                    __fadd_rn(v.z, ev.z), __fadd_rn(v.w, ev.w));
                }
                const uint4 rnd = philox10(philox_counter(q, a.step, (uint32_t)w), a.rk);
                const int c0 = quantize_tma<LEVELS>(v.x, aq, a, rnd.x);
                const int c1 = quantize_tma<LEVELS>(v.y, aq, a, rnd.y);
                const int c2 = quantize_tma<LEVELS>(v.z, aq, a, rnd.z);
                const int c3 = quantize_tma<LEVELS>(v.w, aq, a, rnd.w);
                const int v0 = code_value<LEVELS>(c0), v1 = code_value<LEVELS>(c1);
                const int v2 = code_value<LEVELS>(c2), v3 = code_value<LEVELS>(c3);
                s0 += v0;
                s1 += v1;
                s2 += v2;
                s3 += v3;
                if (BITS != 0)
                    pk.store(lane, c0, c1, c2, c3,
                             a.codes + (long long)w * a.row_bytes + blk * (16 * BITS));
                if (EF && a.update_e && in) {
                    float4 en;
                    en.x = __fsub_rn(v.x, __fmul_rn(small_int_to_float(v0), c));
                    en.y = __fsub_rn(v.y, __fmul_rn(small_int_to_float(v1), c));
                    en.z = __fsub_rn(v.z, __fmul_rn(small_int_to_float(v2), c));
                    en.w = __fsub_rn(v.w, __fmul_rn(small_int_to_float(v3), c));
                    __stcs(reinterpret_cast<float4*>(a.e + (long long)w * a.d + j0), en);
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
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8 * s);
    }
}

size_t tma_smem_bytes(int W, bool ef, int stages) {
    const int rows = ef ? 2 * W : W;
    return (size_t)stages * rows * kTmaTile * sizeof(float) + 2 * stages * sizeof(unsigned long long);
}

template <int LEVELS, int BITS, bool EF, int STAGES>
static cudaError_t launch_tma_inst(const QuantArgs& a, int grid, cudaStream_t st) {
    auto kern = quant_tma_kernel<LEVELS, BITS, EF, STAGES>;
    const size_t smem = tma_smem_bytes(a.W, EF, STAGES);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kTmaThreads, smem, st>>>(a);
    return cudaGetLastError();
}

template <int LEVELS, bool EF, int STAGES>
static cudaError_t launch_tma_bits(const QuantArgs& a, int bits, int grid, cudaStream_t st) {
    switch (bits) {
        case 0: return launch_tma_inst<LEVELS, 0, EF, STAGES>(a, grid, st);
        case 4: return launch_tma_inst<LEVELS, 4, EF, STAGES>(a, grid, st);
        case 5: return launch_tma_inst<LEVELS, 5, EF, STAGES>(a, grid, st);
        case 8: return launch_tma_inst<LEVELS, 8, EF, STAGES>(a, grid, st);
        default: return launch_tma_inst<LEVELS, 16, EF, STAGES>(a, grid, st);
    }
}

cudaError_t launch_quant_tma(const QuantArgs& a, int levels, int bits, bool ef, int stages,
                             int grid, cudaStream_t st) {
#define GQ_TMA(LV, E)                                                            \
    (stages == 2 ? launch_tma_bits<LV, E, 2>(a, bits, grid, st)                  \
                 : stages == 3 ? launch_tma_bits<LV, E, 3>(a, bits, grid, st)    \
                               : launch_tma_bits<LV, E, 4>(a, bits, grid, st))
    if (levels == 0) return ef ? GQ_TMA(0, true) : GQ_TMA(0, false);
    return ef ? GQ_TMA(1, true) : GQ_TMA(1, false);
#undef GQ_TMA
}

}  // namespace gq
