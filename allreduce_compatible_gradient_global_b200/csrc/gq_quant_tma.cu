// gq_quant_tma.cu -- the fused second pass (steps 2-5) with the worker rows
// staged in shared memory by bulk asynchronous copies (sm_100a).
//
// Why: the pass is bound by how many bytes are in flight while the SM spends
// ~20 instructions per element on Philox, rounding and packing.  Holding the
// in-flight rows in registers (one float4 per worker per lane) caps the
// resident warps; here a producer warp streams each worker's row segment of
// a 1024-coordinate tile with one cp.async.bulk into a ring of `stages` tiles,
// and eight compute warps read their 128-coordinate block of every row from
// shared memory.  The copies run ahead by stages - 1 tiles regardless of how
// long the compute takes.
//
// Synchronization: per stage a "full" mbarrier (one producer arrival plus the
// transaction bytes of the copies) and an "empty" mbarrier (one arrival per
// compute warp).  Every wait is bounded by the global timer; on expiry the
// waiting warp raises a flag in the workspace and leaves its loop, and the
// producer drains the copies it issued before the block exits.
//
// Arithmetic, packing and outputs are those of quant_kernel, bit for bit.
//
// Exponential levels take a shorter road to the same codes.  r = fl(v a) is
// scaled by 2^(L-127) rounding toward zero, which puts the finest level
// 2^-(L-1) on 2^-126: a level's index becomes the biased exponent field, and
// the bottom bracket [0, 2^-(L-1)) becomes the subnormal range, whose mantissa
// is floor(p 2^23) with p = |r| 2^(L-1).  Adding the 23 random bits to the bit
// pattern carries out of the mantissa exactly on the round-up event in every
// bracket, the bottom one included, so one integer add and one mask give the
// rounded level as a float (+-2^(idx-127), or +-0), and the top nine bits
// (sign, exponent) index a 512-entry table of signed codes in shared memory.
//
// Philox: with W known at compile time (W = 8), the workers' halves of the
// first two rounds (philox10_split) are computed once per block into shared
// memory, and each coordinate block's half is shared by the W workers.  On
// the uniform pass the executed instructions barely change (20.94 per element
// against 20.71: one more 16-byte shared load per worker and block), but the
// FMA-heavy pipe, which carries the multiplies, is busy 58.8% of cycles
// instead of 60.9%, and the pass runs 0.9-1.4% faster (codes bit-identical).
//
// Tile order: block b starts with tile b, then its producer claims each next
// tile from a counter in the workspace header (tiles grid, grid + 1, ...), so
// every block works inside the same narrow window of the rows however unevenly
// the blocks progress (measured on W = 8 rows of 2^26 to 2^30 coordinates: 3-4%
// faster than block b taking tiles b, b + grid, b + 2 grid, ...).  Taking the
// first tile without a claim keeps the claim's round trip out of the first
// copy (8 x 2^16 coordinates, one tile per block: 14.4 us per step against
// 15.3 us; no change at 8 x 25.6 M).  The last producer to finish puts the
// counter back to zero, so two launches must not share a workspace at the
// same time.  The per-bucket instantiation keeps the static order: it
// prefetches the next block's scale a tile ahead.
#include <cfloat>
#include <type_traits>

#include "gq_internal.h"
#include "gq_pdl.cuh"

namespace gq {

constexpr int kTmaTile = 1024;  // coordinates per worker row per stage
constexpr int kTmaComputeWarps = kTmaTile / 128;
constexpr int kTmaThreads = (kTmaComputeWarps + 1) * 32;
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s

// Blocks per SM the register budget is cut for (two 3-stage rings of eight
// rows fit one SM's shared memory), and whether W = 8 gets its own fully
// unrolled instantiation.
#ifndef GQ_TMA_MIN_BLOCKS
#define GQ_TMA_MIN_BLOCKS 2
#endif
#ifndef GQ_TMA_SPECIALIZE_W8
#define GQ_TMA_SPECIALIZE_W8 1
#endif

// Whole tiles (all but a ragged last one) take a copy of the block body
// without coordinate checks: 3-5% faster on the GPT-2-sized and 8 x 2^26
// workloads, even elsewhere.  Not with error feedback: that pass is bound by
// HBM, measured no gain, and the second copy of its body would spill within
// two blocks' registers.
// The exponential-level code table: signed bytes at a fixed shared address, so
// the top nine bits of a rounded level index it with no scaling (1.05 ms
// against 1.12 ms for 32-bit entries after the ring, GPT-2-sized workload).
constexpr int kExpTableSize = 512;
// Dynamic shared memory after the ring: 2 * stages mbarriers and a tile number
// per stage, room for at most kMaxStages.
constexpr int kMaxStages = 8;
constexpr size_t kTmaTailBytes =
    2 * kMaxStages * sizeof(unsigned long long) + kMaxStages * sizeof(long long);

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

// One bounded try: the thread may be suspended (issuing nothing) until the
// phase completes or about kSuspendHintNs pass, whichever comes first.
constexpr uint32_t kSuspendHintNs = 100000u;
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(kSuspendHintNs)
        : "memory");
    return ok != 0;
}

// Wait for the phase with the given parity to complete, for at most
// limit_ns; false (and the flag raised) if it never did.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, WsHeader* hdr,
                                                  unsigned long long limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_ns() - t0 > limit_ns) {
            atomicOr(&hdr->flags, kFlagPipelineTimeout);
            return false;
        }
    }
    return true;
}

// Self-test of the bounded wait: one thread waits on an mbarrier that nothing
// will ever complete (the first phase of a barrier expecting one arrival that
// never comes), gives up after limit_ns and raises the timeout flag, exactly
// as a stalled pipeline would.  Nothing faults and the context stays usable.
__global__ void wait_timeout_selftest_kernel(WsHeader* hdr, unsigned long long limit_ns) {
    __shared__ __align__(8) unsigned long long bar;
    if (threadIdx.x != 0) return;
    const uint32_t b = smem_addr(&bar);
    mbar_init(b, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    mbar_wait_bounded(b, 0u, hdr, limit_ns);
}

cudaError_t launch_wait_timeout_selftest(WsHeader* hdr, unsigned long long limit_ns,
                                         cudaStream_t st) {
    wait_timeout_selftest_kernel<<<1, 32, 0, st>>>(hdr, limit_ns);
    return cudaGetLastError();
}

// One bulk copy global -> shared (no multicast), completing on `bar`.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(dst), "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// Signed code of a rounded exponential level from its top nine bits h
// (sign, biased exponent): the exponent field is the level index once the
// finest level sits on 2^-126.  Fields past L (only reachable from a
// non-finite input, which also raises the scale flag) give code 0.
__device__ __forceinline__ int exp_table_entry(int h, int L) {
    const int e = h & 255;
    const int idx = e <= L ? e : 0;
    return (h >> 8) ? -idx : idx;
}

// WT: the number of workers when known at compile time (the worker loop is
// then fully unrolled and the Philox chains of all workers interleave), or 0.
template <int LEVELS, int BITS, bool EF, int WT, bool BQ, bool WOFF>
__global__ void __launch_bounds__(kTmaThreads, GQ_TMA_MIN_BLOCKS)
    quant_tma_kernel(const __grid_constant__ QuantArgs a, int stages) {
    extern __shared__ __align__(128) unsigned char smem[];
    // per-bucket scales are prefetched one tile ahead in the static order
    constexpr bool kDynamic = !BQ;
    const int W = WT > 0 ? WT : a.W;
    const int rows = EF ? 2 * W : W;  // g rows, then e rows
    float* buf = reinterpret_cast<float*>(smem);
    unsigned long long* bars = reinterpret_cast<unsigned long long*>(
        smem + (size_t)stages * rows * kTmaTile * sizeof(float));
    long long* tile_of = reinterpret_cast<long long*>(bars + 2 * kMaxStages);
    __shared__ signed char code_table[kExpTableSize];
    const uint32_t full0 = smem_addr(bars);
    const uint32_t empty0 = smem_addr(bars + stages);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long ntiles = (a.d + kTmaTile - 1) / kTmaTile;
    const long long nblk = (a.d + 127) >> 7;

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, kTmaComputeWarps);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (LEVELS != 0 && BITS != 0)
        for (int h = threadIdx.x; h < kExpTableSize; h += kTmaThreads)
            code_table[h] = exp_table_entry(h, a.L);  // |code| <= 15
    // everything above touched shared memory only: now wait for the previous
    // kernel in the stream (the norm pass) and let the next one be scheduled
    pdl_wait();
    pdl_launch_dependents();
    // The unrolled kernel's workers' halves of Philox's first two rounds, once
    // per block (philox10_split); each coordinate block's half is shared by
    // all WT workers.
    __shared__ uint4 worker_part[WT > 0 ? WT : 1];
    if (WT > 0 && threadIdx.x < WT) {
        const uint32_t st = a.step_dev ? __ldg(a.step_dev) : a.step;
        const uint32_t wid = WOFF ? a.worker0 + threadIdx.x : threadIdx.x;
        const PhiloxWorkerPart p = philox_worker_part(st, wid, a.rk);
        worker_part[threadIdx.x] = make_uint4(p.bx, p.hz, p.lw, 0u);
    }
    __syncthreads();

    if (warp == kTmaComputeWarps) {
        // ---------------- producer: one lane issues every copy ----------------
        if (lane == 0) {
            // stage s of round `round` holds this CTA's k-th tile, k = round * stages + s
            int s = 0;
            uint32_t round = 0;
            long long issued = 0;
            bool ok = true;
            // the first tile is the block's own (the grid never exceeds the tile
            // count), so the first copy waits for no claim; later tiles are
            // claimed beyond the first wave
            long long t = blockIdx.x;
            for (;; ++issued) {
                if (!kDynamic && t >= ntiles) break;
                if (round > 0 && !mbar_wait_bounded(empty0 + 8 * s, (round - 1) & 1u, a.hdr)) {
                    ok = false;
                    break;
                }
                if (kDynamic && t >= ntiles) {  // no tile left: tell the compute warps
                    tile_of[s] = -1;
                    mbar_arrive(full0 + 8 * s);
                    break;
                }
                const long long j0 = t * kTmaTile;
                // claim the next tile now, so the atomic's round trip overlaps this one
                const long long t_next =
                    kDynamic ? (long long)gridDim.x + atomicAdd(&a.hdr->tile_next, 1u)
                             : t + gridDim.x;
                tile_of[s] = t;
                const long long n = a.d - j0 < kTmaTile ? a.d - j0 : kTmaTile;
                const uint32_t bytes = (uint32_t)(n * sizeof(float));
                mbar_arrive_expect_tx(full0 + 8 * s, bytes * (uint32_t)rows);
                for (int r = 0; r < rows; ++r) {
                    const float* src = (r < W ? a.g + (long long)r * a.d
                                              : a.e + (long long)(r - W) * a.d) + j0;
                    bulk_g2s(smem_addr(buf + ((size_t)s * rows + r) * kTmaTile), src, bytes,
                             full0 + 8 * s);
                }
                t = t_next;
                if (++s == stages) {
                    s = 0;
                    ++round;
                }
            }
            // Drain: every issued stage must have landed before the block exits.
            // On the normal path the consumers already waited for all of them;
            // after a timeout, wait (bounded) for the last `stages` issued tiles.
            if (!ok) {
                const long long first = issued > stages ? issued - stages : 0;
                for (long long k = first; k < issued; ++k)
                    mbar_wait_bounded(full0 + 8 * (int)(k % stages), (uint32_t)((k / stages) & 1),
                                      a.hdr);
            }
            if (kDynamic) {
                // The last producer to finish claiming resets the counters for the
                // next launch on this workspace (stream order publishes them).
                __threadfence();
                if (atomicAdd(&a.hdr->tile_done, 1u) == gridDim.x - 1) {
                    atomicExch(&a.hdr->tile_next, 0u);
                    atomicExch(&a.hdr->tile_done, 0u);
                }
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
            aq = okS ? __fdiv_rd(a.smax, S) : 0.f;  // |v| aq <= s for every |v| <= S
            c = __fdiv_rn(S, a.smax);
        } else {
            aq = okS ? __fdiv_rd(1.0f, S) : 0.f;  // |v| aq <= 1 for every |v| <= S
            c = __fmul_rn(S, a.finest);
        }
    }
    const uint32_t step = a.step_dev ? __ldg(a.step_dev) : a.step;
    Packer<BITS> pk;
    pk.init(lane);
    const long long row_bytes = a.row_bytes;
    int s = 0;
    uint32_t phase = 0;
    // per-bucket scales: this warp's next block's multiplier and unit, loaded
    // one tile ahead so that the load's latency hides behind a tile of work
    float aq_next = 0.f, c_next = 0.f;
    const long long blk_step = (long long)gridDim.x * kTmaComputeWarps;
    if (BQ) {
        const long long b0 = (long long)blockIdx.x * kTmaComputeWarps + warp;
        if (b0 < nblk) {
            aq_next = __ldg(a.bq_mult + (b0 >> a.bucket_shift));
            c_next = __ldg(a.bq_unit + (b0 >> a.bucket_shift));
        }
    }
    for (long long tt = blockIdx.x;; tt += gridDim.x) {
        if (!kDynamic && tt >= ntiles) break;
        if (!mbar_wait_bounded(full0 + 8 * s, phase, a.hdr)) break;
        const long long t = kDynamic ? tile_of[s] : tt;
        if (t < 0) break;  // the producer found no tile left
        const long long blk = t * kTmaComputeWarps + warp;
        // FULL: every coordinate of the tile exists (no bounds checks)
        auto block_body = [&](auto full_tag) {
            constexpr bool FULL = decltype(full_tag)::value;
            if (BQ) {  // per-bucket scale of this block
                aq = aq_next;
                c = c_next;
                const long long bn = blk + blk_step;
                if (bn < nblk) {
                    aq_next = __ldg(a.bq_mult + (bn >> a.bucket_shift));
                    c_next = __ldg(a.bq_unit + (bn >> a.bucket_shift));
                }
            }
            const long long j0 = (blk << 7) + (lane << 2);
            const bool in = FULL || j0 < a.d;  // d % 4 == 0: all four or none
            // WOFF = 0: no worker or coordinate offset (the common case)
            const unsigned long long q =
                (unsigned long long)(blk << 5) + (unsigned)lane + (WOFF ? a.q0 : 0ull);
            const float* stage = buf + (size_t)s * rows * kTmaTile + warp * 128 + lane * 4;
            unsigned char* codes_blk = a.codes + blk * (16 * BITS);
            const PhiloxBlockPart bpart =
                WT > 0 ? philox_block_part(q, a.rk) : PhiloxBlockPart{0u, 0u, 0u};
            // uniform levels accumulate the biased patterns (code + kCodeBias);
            // exponential levels accumulate the rounded levels as floats in
            // units of 2^-126 per finest level (exact: integers below 2^24
            // times 2^-126, subnormal or not)
            uint32_t s0 = 0, s1 = 0, s2 = 0, s3 = 0;
            uint32_t p0 = 0, p1 = 0, p2 = 0, p3 = 0;  // an even worker's patterns
            float f0 = 0.f, f1 = 0.f, f2 = 0.f, f3 = 0.f;
#pragma unroll
            for (int w = 0; w < (WT > 0 ? WT : a.W); ++w) {
                float4 v = in ? *reinterpret_cast<const float4*>(stage + (size_t)w * kTmaTile)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
                if (EF && in) {
                    const float4 ev =
                        *reinterpret_cast<const float4*>(stage + (size_t)(W + w) * kTmaTile);
                    v = make_float4(__fadd_rn(v.x, ev.x), __fadd_rn(v.y, ev.y),
                                    __fadd_rn(v.z, ev.z), __fadd_rn(v.w, ev.w));
                }
                // WOFF = 0: the worker word is the loop constant w (the common case)
                const uint32_t wid = WOFF ? a.worker0 + (uint32_t)w : (uint32_t)w;
                uint4 rnd;
                if (WT > 0) {
                    const uint4 wp = worker_part[WT > 0 ? w : 0];
                    rnd = philox10_split(bpart, PhiloxWorkerPart{wp.x, wp.y, wp.z}, a.rk);
                } else {
                    rnd = philox10(philox_counter(q, step, wid), a.rk);
                }
                unsigned char* cdst = codes_blk + (long long)w * row_bytes;
                float4 qv;  // the values Q(v) in units of c, as floats
                if (LEVELS == 0) {
                    const float t0 = quant_uniform_biased_unclamped(v.x, aq, rnd.x);
                    const float t1 = quant_uniform_biased_unclamped(v.y, aq, rnd.y);
                    const float t2 = quant_uniform_biased_unclamped(v.z, aq, rnd.z);
                    const float t3 = quant_uniform_biased_unclamped(v.w, aq, rnd.w);
                    const uint32_t b0 = __float_as_uint(t0), b1 = __float_as_uint(t1);
                    const uint32_t b2 = __float_as_uint(t2), b3 = __float_as_uint(t3);
                    // the unrolled kernel adds two workers' patterns per
                    // three-input add (the sums are mod 2^32, so exact in any
                    // order): 3% faster than one add per worker
                    if (WT > 0 && WT % 2 == 0) {
                        if ((w & 1) == 0) {
                            p0 = b0;
                            p1 = b1;
                            p2 = b2;
                            p3 = b3;
                        } else {
                            s0 += p0 + b0;
                            s1 += p1 + b1;
                            s2 += p2 + b2;
                            s3 += p3 + b3;
                        }
                    } else {
                        s0 += b0;
                        s1 += b1;
                        s2 += b2;
                        s3 += b3;
                    }
                    if (BITS != 0) pk.template store<kCodeBias>(lane, b0, b1, b2, b3, cdst);
                    if (EF) {
                        qv.x = __fsub_rn(t0, 12582912.0f);
                        qv.y = __fsub_rn(t1, 12582912.0f);
                        qv.z = __fsub_rn(t2, 12582912.0f);
                        qv.w = __fsub_rn(t3, 12582912.0f);
                    }
                } else {
                    const uint32_t y0 = exp_round_bits(v.x, aq, a.exp_shift, rnd.x);
                    const uint32_t y1 = exp_round_bits(v.y, aq, a.exp_shift, rnd.y);
                    const uint32_t y2 = exp_round_bits(v.z, aq, a.exp_shift, rnd.z);
                    const uint32_t y3 = exp_round_bits(v.w, aq, a.exp_shift, rnd.w);
                    const float q0 = __uint_as_float(y0 & 0xFF800000u);
                    const float q1 = __uint_as_float(y1 & 0xFF800000u);
                    const float q2 = __uint_as_float(y2 & 0xFF800000u);
                    const float q3 = __uint_as_float(y3 & 0xFF800000u);
                    f0 = __fadd_rn(f0, q0);
                    f1 = __fadd_rn(f1, q1);
                    f2 = __fadd_rn(f2, q2);
                    f3 = __fadd_rn(f3, q3);
                    if (BITS != 0)  // y >> 23 < 512: always inside the table
                        pk.store(lane, code_table[y0 >> 23], code_table[y1 >> 23],
                                 code_table[y2 >> 23], code_table[y3 >> 23], cdst);
                    if (EF) {  // value in units of the finest level (exact)
                        qv.x = __fmul_rn(q0, 0x1p126f);
                        qv.y = __fmul_rn(q1, 0x1p126f);
                        qv.z = __fmul_rn(q2, 0x1p126f);
                        qv.w = __fmul_rn(q3, 0x1p126f);
                    }
                }
                if (EF && a.update_e && in) {
                    float4 en;
                    en.x = __fsub_rn(v.x, __fmul_rn(qv.x, c));
                    en.y = __fsub_rn(v.y, __fmul_rn(qv.y, c));
                    en.z = __fsub_rn(v.z, __fmul_rn(qv.z, c));
                    en.w = __fsub_rn(v.w, __fmul_rn(qv.w, c));
                    __stcs(reinterpret_cast<float4*>(a.e + (long long)w * a.d + j0), en);
                }
            }
            if (LEVELS == 0) {
                const uint32_t off = (uint32_t)W * kCodeBias;
                s0 -= off;
                s1 -= off;
                s2 -= off;
                s3 -= off;
            } else {  // level-value sums to integer units of the finest level
                s0 = (uint32_t)float_units_to_int(f0);
                s1 = (uint32_t)float_units_to_int(f1);
                s2 = (uint32_t)float_units_to_int(f2);
                s3 = (uint32_t)float_units_to_int(f3);
            }
            if (a.sum) store_sum<FULL>(a.sum, a.wire, j0, a.d, (int)s0, (int)s1, (int)s2, (int)s3);
            if (a.out) {
                float4 o;
                o.x = decode_mean((int)s0, c, a.inv_w, a.w_pow2, W);
                o.y = decode_mean((int)s1, c, a.inv_w, a.w_pow2, W);
                o.z = decode_mean((int)s2, c, a.inv_w, a.w_pow2, W);
                o.w = decode_mean((int)s3, c, a.inv_w, a.w_pow2, W);
                store_out4<FULL>(a.out, j0, a.d, o);
            }
        };
        if (!EF && (t + 1) * kTmaTile <= a.d)
            block_body(std::true_type{});
        else if (blk < nblk)
            block_body(std::false_type{});
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8 * s);
        if (++s == stages) {
            s = 0;
            phase ^= 1u;
        }
    }
}

size_t tma_smem_bytes(int W, bool ef, int stages) {
    const int rows = ef ? 2 * W : W;
    return (size_t)stages * rows * kTmaTile * sizeof(float) + kTmaTailBytes;
}

template <int LEVELS, int BITS, bool EF, int WT, bool BQ, bool WOFF>
static cudaError_t launch_tma_inst(const QuantArgs& a, int stages, int grid, cudaStream_t st) {
    auto kern = quant_tma_kernel<LEVELS, BITS, EF, WT, BQ, WOFF>;
    const size_t smem = tma_smem_bytes(a.W, EF, stages);
    static int limits[64] = {};
    cudaError_t e = ensure_dynamic_smem((const void*)kern, smem, limits);
    if (e != cudaSuccess) return e;
    return launch_with_pdl(kern, dim3(grid), dim3(kTmaThreads), smem, st, pdl_allowed(st), a,
                           stages);
}

template <int LEVELS, int BITS, bool EF>
static cudaError_t launch_tma_w(const QuantArgs& a, int stages, int grid, cudaStream_t st) {
    // per-bucket scales get their own instantiations, so the global-scale
    // kernel keeps one multiplier in a register for the whole launch
    // The unrolled W = 8 kernel gets the worker and coordinate offsets of a
    // data-parallel rank or chunk as a separate instantiation; the general one
    // always adds them.
    const bool woff = a.worker0 != 0 || a.q0 != 0;
    if (a.bq_mult) {
        if (GQ_TMA_SPECIALIZE_W8 && a.W == 8)
            return woff ? launch_tma_inst<LEVELS, BITS, EF, 8, true, true>(a, stages, grid, st)
                        : launch_tma_inst<LEVELS, BITS, EF, 8, true, false>(a, stages, grid, st);
        return launch_tma_inst<LEVELS, BITS, EF, 0, true, true>(a, stages, grid, st);
    }
    if (GQ_TMA_SPECIALIZE_W8 && a.W == 8)
        return woff ? launch_tma_inst<LEVELS, BITS, EF, 8, false, true>(a, stages, grid, st)
                    : launch_tma_inst<LEVELS, BITS, EF, 8, false, false>(a, stages, grid, st);
    return launch_tma_inst<LEVELS, BITS, EF, 0, false, true>(a, stages, grid, st);
}

template <int LEVELS, bool EF>
static cudaError_t launch_tma_bits(const QuantArgs& a, int bits, int stages, int grid,
                                   cudaStream_t st) {
    switch (bits) {
        case 0: return launch_tma_w<LEVELS, 0, EF>(a, stages, grid, st);
        case 4: return launch_tma_w<LEVELS, 4, EF>(a, stages, grid, st);
        case 5: return launch_tma_w<LEVELS, 5, EF>(a, stages, grid, st);
        case 8: return launch_tma_w<LEVELS, 8, EF>(a, stages, grid, st);
        default: return launch_tma_w<LEVELS, 16, EF>(a, stages, grid, st);
    }
}

cudaError_t launch_quant_tma(const QuantArgs& a, int levels, int bits, bool ef, int stages,
                             int grid, cudaStream_t st) {
    if (levels == 0)
        return ef ? launch_tma_bits<0, true>(a, bits, stages, grid, st)
                  : launch_tma_bits<0, false>(a, bits, stages, grid, st);
    return ef ? launch_tma_bits<1, true>(a, bits, stages, grid, st)
              : launch_tma_bits<1, false>(a, bits, stages, grid, st);
}

}  // namespace gq
