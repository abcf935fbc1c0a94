// gq_psgd.cu -- PowerSGD low-rank step for LQ-SGD (sm_100a).
//
// "Trustworthy Efficient Communication for Distributed Learning using LQ-SGD
// Algorithm" (review, "What carries the argument"): G ~ P Q^T by PowerSGD's
// low-rank step, P and Q log-quantized before their All-Reduce, error
// E_t = G'_t - Ghat_t added back on the next step.  Per matrix (n x m, rank r
// <= 8) and worker w, with the previous step's P_hat and mean Q as state:
//
//   project        E_w = M_prev,w - P_hat Q^T (deferred error; skipped on the
//                  first step), M_w = G_w + E_w (written back as the state),
//                  P_w = M_w Q
//   orthonormalize P_hat = MGS(sum_w decode(LQ(P_w)))  (in place, fp64 sums)
//   back_project   Q_w = M_w^T P_hat  (per row-chunk partials, then a
//                  fixed-order sum over chunks)
//   mean           Q = fl(sum_w decode(LQ(Q_w)) / W)
//   reconstruct    Ghat = P_hat Q^T
//
// Nothing here is a dense contraction worth tensor cores: with r <= 8 every
// pass streams the n x m matrices once at r (or 2r) FMAs per element, which is
// HBM-bound on the CUDA cores.  The element-wise formulas are fixed so that the
// state is reproducible: Ghat_ij = fma chain over k of P_hat[i,k] Q[j,k] from 0,
// E = fl(M_prev - Ghat_ij), M = fl(G + E).
#include <cfloat>

#include "gq_psgd.h"

namespace gq {

constexpr int kPsgdThreads = 256;
constexpr int kProjRowsPerWarp = 2;
constexpr int kProjRowsPerTile = kProjRowsPerWarp * (kPsgdThreads / 32);  // 16
constexpr int kBackColsPerTile = 4 * kPsgdThreads;                        // 1024 (VEC)

// The matrix of a work tile: tile0[] holds each matrix's first tile.
__device__ __forceinline__ int matrix_of(const PsgdArgs& a, long long t) {
    int lo = 0, hi = a.count - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (a.tile0[mid] <= t) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// Per-lane asynchronous 16-byte copies global -> shared (bypassing L1), so
// that several loads per lane stay in flight without holding registers.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
    const unsigned d = (unsigned)__cvta_generic_to_shared(smem_dst);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Projection pass: resident blocks per SM by rank (the register budget the
// kernels are cut for; the 4r-float Q slice per column group grows with r).
template <int R>
struct ProjCfg {
    static constexpr int min_blocks = R <= 2 ? 4 : (R <= 4 ? 3 : 2);
};
constexpr int kBackStages = 8;  // per-thread pipeline depth of the back projection

template <int R>
__device__ __forceinline__ float lowrank_value(const float (&p)[R], const float* q) {
    float acc = 0.f;
#pragma unroll
    for (int k = 0; k < R; ++k) acc = __fmaf_rn(p[k], q[k], acc);
    return acc;
}

// ---------------------------------------------------------------------------
// project, any m: tiles of (matrix, worker, 16 rows); each warp takes two rows
// and its lanes stride over the columns one float at a time.  P_w[i,k] sums
// lane-sequential partials, then a xor butterfly over the warp.  (When every m
// is a multiple of 4, psgd_project_q_kernel below takes the pass.)
// ---------------------------------------------------------------------------
template <int R, bool HAVE_PREV>
__global__ void __launch_bounds__(kPsgdThreads, ProjCfg<R>::min_blocks)
    psgd_project_kernel(const __grid_constant__ PsgdArgs a) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (long long t = blockIdx.x; t < a.tile0[a.count]; t += gridDim.x) {
        const int l = matrix_of(a, t);
        const long long lt = t - a.tile0[l];
        const int n = a.rows[l], m = a.cols[l];
        const long long row_tiles = (n + kProjRowsPerTile - 1) / kProjRowsPerTile;
        const int w = (int)(lt / row_tiles);
        const int i0 = (int)(lt - (long long)w * row_tiles) * kProjRowsPerTile +
                       warp * kProjRowsPerWarp;
        if (i0 >= n) continue;
        const bool two = i0 + 1 < n;
        const long long base = (long long)w * a.total + a.goff[l];
        const float* g0 = a.g + base + (long long)i0 * m;
        float* m0 = a.m + base + (long long)i0 * m;
        const float* qm = a.q + a.qoff[l];
        float p0[R], p1[R];
        if (HAVE_PREV) {
            const float* pr = a.p + a.poff[l] + (long long)i0 * R;
#pragma unroll
            for (int k = 0; k < R; ++k) {
                p0[k] = __ldg(pr + k);
                p1[k] = two ? __ldg(pr + R + k) : 0.f;
            }
        }
        float acc0[R], acc1[R];
#pragma unroll
        for (int k = 0; k < R; ++k) acc0[k] = acc1[k] = 0.f;
        for (int j = lane; j < m; j += 32) {
            float q[R];
#pragma unroll
            for (int k = 0; k < R; ++k) q[k] = __ldg(qm + (long long)j * R + k);
            float eA = m0[j], eB = two ? m0[m + j] : 0.f;
            if (HAVE_PREV) {
                eA = __fsub_rn(eA, lowrank_value<R>(p0, q));
                eB = __fsub_rn(eB, lowrank_value<R>(p1, q));
            }
            const float vA = __fadd_rn(g0[j], eA);
            const float vB = two ? __fadd_rn(g0[m + j], eB) : 0.f;
            m0[j] = vA;
            if (two) m0[m + j] = vB;
#pragma unroll
            for (int k = 0; k < R; ++k) {
                acc0[k] = __fmaf_rn(vA, q[k], acc0[k]);
                acc1[k] = __fmaf_rn(vB, q[k], acc1[k]);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
            for (int k = 0; k < R; ++k) {
                acc0[k] = __fadd_rn(acc0[k], __shfl_xor_sync(kFull, acc0[k], o));
                acc1[k] = __fadd_rn(acc1[k], __shfl_xor_sync(kFull, acc1[k], o));
            }
        }
        if (lane == 0) {
            float* pw = a.pw + (long long)w * a.ptotal + a.poff[l] + (long long)i0 * R;
#pragma unroll
            for (int k = 0; k < R; ++k) {
                pw[k] = acc0[k];
                if (two) pw[R + k] = acc1[k];
            }
        }
    }
}

// ---------------------------------------------------------------------------
// project, every m a multiple of 4 (any rank): the same arithmetic and
// summation order as psgd_project_kernel, with columns taken as float4 groups
// (lane-sequential partials over j4 = lane + 32 it, four columns each) and the
// Q slice of each column step staged once per block.  All 8 warps of a block walk the same column
// groups (j4 = lane + 32 it) of their own two rows, so one copy of Q's rows
// 4 j4 .. 4 j4 + 3 serves the block instead of being re-read by every row
// pair through L1.  Ring of kQStages slots: per warp the lane-private G / M
// vectors, per block the shared Q slice; one block barrier per step makes the
// step's copies visible and frees the slot the previous step read.
// ---------------------------------------------------------------------------
constexpr int kQStages = 3;

template <int R, bool HAVE_PREV>
__global__ void __launch_bounds__(kPsgdThreads, ProjCfg<R>::min_blocks)
    psgd_project_q_kernel(const __grid_constant__ PsgdArgs a) {
    extern __shared__ float4 qsm[];
    float4* qring = qsm;                                    // [kQStages][32 * R]
    float4* vring = qsm + kQStages * 32 * R;                // [8 warps][kQStages][4][32]
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float4* ring = vring + (size_t)warp * kQStages * 4 * 32;
    for (long long t = blockIdx.x; t < a.tile0[a.count]; t += gridDim.x) {
        const int l = matrix_of(a, t);
        const long long lt = t - a.tile0[l];
        const int n = a.rows[l], m = a.cols[l];
        const long long row_tiles = (n + kProjRowsPerTile - 1) / kProjRowsPerTile;
        const int w = (int)(lt / row_tiles);
        const int i0 = (int)(lt - (long long)w * row_tiles) * kProjRowsPerTile +
                       warp * kProjRowsPerWarp;
        const bool row0 = i0 < n, two = i0 + 1 < n;  // warp-uniform
        const long long base = (long long)w * a.total + a.goff[l];
        const float* g0 = a.g + base + (long long)(row0 ? i0 : 0) * m;
        float* m0 = a.m + base + (long long)(row0 ? i0 : 0) * m;
        const float* qm = a.q + a.qoff[l];
        float p0[R], p1[R];
        if (HAVE_PREV) {
            const float* pr = a.p + a.poff[l] + (long long)(row0 ? i0 : 0) * R;
#pragma unroll
            for (int k = 0; k < R; ++k) {
                p0[k] = row0 ? __ldg(pr + k) : 0.f;
                p1[k] = two ? __ldg(pr + R + k) : 0.f;
            }
        }
        float acc0[R], acc1[R];
#pragma unroll
        for (int k = 0; k < R; ++k) acc0[k] = acc1[k] = 0.f;
        const float4* gA4 = reinterpret_cast<const float4*>(g0);
        const float4* mA4 = reinterpret_cast<const float4*>(m0);
        const float4* gB4 = reinterpret_cast<const float4*>(g0 + m);
        const float4* mB4 = reinterpret_cast<const float4*>(m0 + m);
        const int m4 = m >> 2;
        const int nit = (m4 + 31) / 32;  // the same for every warp of the block
        // thread x < 32 R copies float4 k = x % R of the Q rows of lane x / R
        const int qx = threadIdx.x, ql = qx / R, qk = qx - ql * R;
        auto issue = [&](int it) {
            const int slot = it % kQStages;
            const int j4 = lane + it * 32;
            if (row0 && j4 < m4) {
                float4* d = ring + slot * 128 + lane;
                cp_async16(d, gA4 + j4);
                cp_async16(d + 32, mA4 + j4);
                if (two) {
                    cp_async16(d + 64, gB4 + j4);
                    cp_async16(d + 96, mB4 + j4);
                }
            }
            const int qj4 = ql + it * 32;
            if (qx < 32 * R && qj4 < m4)
                cp_async16(qring + slot * 32 * R + qx,
                           reinterpret_cast<const float4*>(qm + (long long)qj4 * 4 * R) + qk);
        };
        __syncthreads();  // the previous tile's reads of the rings are done
#pragma unroll
        for (int it = 0; it < kQStages - 1; ++it) {
            if (it < nit) issue(it);
            cp_async_commit();
        }
        for (int it = 0; it < nit; ++it) {
            cp_async_wait<kQStages - 2>();  // this thread's copies of step `it` landed
            __syncthreads();                // ... and every thread's; slot (it - 1) is free
            if (it + kQStages - 1 < nit) issue(it + kQStages - 1);
            cp_async_commit();
            const int j4 = lane + it * 32;
            if (!row0 || j4 >= m4) continue;
            const int slot = it % kQStages;
            float q[4 * R];  // rows 4 j4 .. 4 j4 + 3 of Q, R values each
            const float4* qs = qring + slot * 32 * R + lane * R;
#pragma unroll
            for (int k = 0; k < R; ++k) {
                const float4 v = qs[k];
                q[4 * k] = v.x;
                q[4 * k + 1] = v.y;
                q[4 * k + 2] = v.z;
                q[4 * k + 3] = v.w;
            }
            const float4* d = ring + slot * 128 + lane;
            const float4 ga = d[0], ma = d[32];
            float4 gb = make_float4(0.f, 0.f, 0.f, 0.f), mb = gb;
            if (two) {
                gb = d[64];
                mb = d[96];
            }
            const float gA[4] = {ga.x, ga.y, ga.z, ga.w}, mA[4] = {ma.x, ma.y, ma.z, ma.w};
            const float gB[4] = {gb.x, gb.y, gb.z, gb.w}, mB[4] = {mb.x, mb.y, mb.z, mb.w};
            float outA[4], outB[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float* qc = q + c * R;
                float eA = mA[c], eB = mB[c];
                if (HAVE_PREV) {
                    eA = __fsub_rn(eA, lowrank_value<R>(p0, qc));
                    eB = __fsub_rn(eB, lowrank_value<R>(p1, qc));
                }
                outA[c] = __fadd_rn(gA[c], eA);
                outB[c] = __fadd_rn(gB[c], eB);
#pragma unroll
                for (int k = 0; k < R; ++k) {
                    acc0[k] = __fmaf_rn(outA[c], qc[k], acc0[k]);
                    acc1[k] = __fmaf_rn(outB[c], qc[k], acc1[k]);
                }
            }
            __stcs(reinterpret_cast<float4*>(m0) + j4, make_float4(outA[0], outA[1], outA[2], outA[3]));
            if (two)
                __stcs(reinterpret_cast<float4*>(m0 + m) + j4,
                       make_float4(outB[0], outB[1], outB[2], outB[3]));
        }
        cp_async_wait<0>();
        if (!row0) continue;  // warp-uniform; no barrier follows before the next tile's
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
            for (int k = 0; k < R; ++k) {
                acc0[k] = __fadd_rn(acc0[k], __shfl_xor_sync(kFull, acc0[k], o));
                acc1[k] = __fadd_rn(acc1[k], __shfl_xor_sync(kFull, acc1[k], o));
            }
        }
        if (lane == 0) {
            float* pw = a.pw + (long long)w * a.ptotal + a.poff[l] + (long long)i0 * R;
#pragma unroll
            for (int k = 0; k < R; ++k) {
                pw[k] = acc0[k];
                if (two) pw[R + k] = acc1[k];
            }
        }
    }
}

// ---------------------------------------------------------------------------
// orthonormalize: one block per matrix, modified Gram-Schmidt over the columns
// in order, fp64 sums in a fixed order, fp32 storage.  A column whose
// remaining norm is 0 stays 0.
// ---------------------------------------------------------------------------
__device__ __forceinline__ double block_sum_psgd(double x, double* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(kFull, x, o);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    __syncthreads();
    if (lane == 0) red[warp] = x;
    __syncthreads();
    double t = 0.0;
    for (int k = 0; k < (int)(blockDim.x >> 5); ++k) t += red[k];
    return t;
}

template <int R>
__global__ void __launch_bounds__(1024) psgd_orth_kernel(const __grid_constant__ PsgdArgs a) {
    __shared__ double red[32];
    const int l = blockIdx.x;
    if (l >= a.count) return;
    const int n = a.rows[l];
    float* P = a.psum + a.poff[l];  // in place
    for (int k = 0; k < R; ++k) {
        double s = 0.0;
        for (int i = threadIdx.x; i < n; i += blockDim.x) {
            const double v = (double)P[(long long)i * R + k];
            s += v * v;
        }
        const double nrm = sqrt(block_sum_psgd(s, red));
        if (nrm > 0.0)
            for (int i = threadIdx.x; i < n; i += blockDim.x)
                P[(long long)i * R + k] = (float)((double)P[(long long)i * R + k] / nrm);
        for (int k2 = k + 1; k2 < R; ++k2) {
            __syncthreads();  // column k is final before it is read by other threads
            double dp = 0.0;
            for (int i = threadIdx.x; i < n; i += blockDim.x)
                dp += (double)P[(long long)i * R + k] * (double)P[(long long)i * R + k2];
            const double dsum = block_sum_psgd(dp, red);
            for (int i = threadIdx.x; i < n; i += blockDim.x) {
                const long long x = (long long)i * R;
                P[x + k2] = (float)((double)P[x + k2] - dsum * (double)P[x + k]);
            }
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// back_project: tiles of (matrix, worker, column tile, row chunk).  Each thread
// owns 4 columns (VEC) or 1 and runs down the chunk's rows, with the chunk's
// P_hat rows staged in shared memory (stride RP, padded to 4).  Writes its
// partial Q_w rows for the chunk; back_reduce sums the chunks in order.
// ---------------------------------------------------------------------------
template <int R>
struct Padded {
    static constexpr int value = (R + 3) & ~3;
};

template <int R, bool VEC>
__global__ void __launch_bounds__(kPsgdThreads)
    psgd_back_kernel(const __grid_constant__ PsgdArgs a) {
    constexpr int RP = Padded<R>::value;
    extern __shared__ float4 smem4[];
    float* ps = reinterpret_cast<float*>(smem4);
    const int cols_per_tile = VEC ? kBackColsPerTile : kPsgdThreads;
    for (long long t = blockIdx.x; t < a.tile0[a.count]; t += gridDim.x) {
        const int l = matrix_of(a, t);
        long long lt = t - a.tile0[l];
        const int n = a.rows[l], m = a.cols[l];
        const int ctiles = (m + cols_per_tile - 1) / cols_per_tile;
        const int chunks = (n + a.chunk_rows - 1) / a.chunk_rows;
        const int c = (int)(lt % chunks);
        lt /= chunks;
        const int ct = (int)(lt % ctiles);
        const int w = (int)(lt / ctiles);
        const int r0 = c * a.chunk_rows;
        const int r1 = min(n, r0 + a.chunk_rows);
        __syncthreads();  // the previous tile's reads of ps are done
        for (int x = threadIdx.x; x < (r1 - r0) * RP; x += kPsgdThreads) {
            const int i = x / RP, k = x - i * RP;
            ps[x] = k < R ? __ldg(a.p + a.poff[l] + (long long)(r0 + i) * R + k) : 0.f;
        }
        __syncthreads();
        const float* mrow = a.m + (long long)w * a.total + a.goff[l];
        float* part = a.qpart + ((long long)c * a.W + w) * a.qtotal + a.qoff[l];
        if (VEC) {
            const int j = ct * kBackColsPerTile + 4 * threadIdx.x;
            if (j < m) {
                // thread-private ring of kBackStages rows of this thread's float4
                float4* ring = reinterpret_cast<float4*>(ps + (size_t)a.chunk_rows * RP);
                const int nrow = r1 - r0;
                const float* src = mrow + (long long)r0 * m + j;
                auto issue = [&](int it) {
                    cp_async16(ring + (it % kBackStages) * kPsgdThreads + threadIdx.x,
                               src + (long long)it * m);
                };
#pragma unroll
                for (int it = 0; it < kBackStages - 1; ++it) {
                    if (it < nrow) issue(it);
                    cp_async_commit();
                }
                float acc[4][R];
#pragma unroll
                for (int cc = 0; cc < 4; ++cc)
#pragma unroll
                    for (int k = 0; k < R; ++k) acc[cc][k] = 0.f;
                for (int it = 0; it < nrow; ++it) {
                    if (it + kBackStages - 1 < nrow) issue(it + kBackStages - 1);
                    cp_async_commit();
                    cp_async_wait<kBackStages - 1>();
                    const float4 v = ring[(it % kBackStages) * kPsgdThreads + threadIdx.x];
                    const float* pr = ps + it * RP;
                    float pk[RP];
#pragma unroll
                    for (int k4 = 0; k4 < RP / 4; ++k4) {
                        const float4 pv = reinterpret_cast<const float4*>(pr)[k4];
                        pk[4 * k4] = pv.x;
                        pk[4 * k4 + 1] = pv.y;
                        pk[4 * k4 + 2] = pv.z;
                        pk[4 * k4 + 3] = pv.w;
                    }
                    const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc)
#pragma unroll
                        for (int k = 0; k < R; ++k)
                            acc[cc][k] = __fmaf_rn(vv[cc], pk[k], acc[cc][k]);
                }
                cp_async_wait<0>();
#pragma unroll
                for (int cc = 0; cc < 4; ++cc)
#pragma unroll
                    for (int k = 0; k < R; ++k) part[(long long)(j + cc) * R + k] = acc[cc][k];
            }
        } else {
            const int j = ct * kPsgdThreads + threadIdx.x;
            if (j < m) {
                float acc[R];
#pragma unroll
                for (int k = 0; k < R; ++k) acc[k] = 0.f;
                for (int i = r0; i < r1; ++i) {
                    const float v = __ldcs(mrow + (long long)i * m + j);
                    const float* pr = ps + (i - r0) * RP;
#pragma unroll
                    for (int k = 0; k < R; ++k) acc[k] = __fmaf_rn(v, pr[k], acc[k]);
                }
#pragma unroll
                for (int k = 0; k < R; ++k) part[(long long)j * R + k] = acc[k];
            }
        }
    }
}

// Q_w = sum over the matrix's row chunks, in chunk order.
__global__ void __launch_bounds__(kPsgdThreads)
    psgd_back_reduce_kernel(const __grid_constant__ PsgdArgs a) {
    for (long long t = blockIdx.x; t < a.tile0[a.count]; t += gridDim.x) {
        const int l = matrix_of(a, t);
        const long long lt = t - a.tile0[l];
        const long long len = (long long)a.cols[l] * a.rank;
        const long long per_w = (len + kPsgdThreads - 1) / kPsgdThreads;
        const int w = (int)(lt / per_w);
        const long long x = (lt - (long long)w * per_w) * kPsgdThreads + threadIdx.x;
        if (x >= len) continue;
        const int chunks = (a.rows[l] + a.chunk_rows - 1) / a.chunk_rows;
        const long long idx = (long long)w * a.qtotal + a.qoff[l] + x;
        float s = a.qpart[idx];
        for (int c = 1; c < chunks; ++c)
            s = __fadd_rn(s, a.qpart[(long long)c * a.W * a.qtotal + idx]);
        a.qw[idx] = s;
    }
}

// Q = fl(Q_sum / W), element-wise over all matrices.
__global__ void psgd_mean_kernel(const float* qsum, float* q, long long len, float W) {
    for (long long x = (long long)blockIdx.x * blockDim.x + threadIdx.x; x < len;
         x += (long long)gridDim.x * blockDim.x)
        q[x] = __fdiv_rn(qsum[x], W);
}

// ---------------------------------------------------------------------------
// reconstruct: Ghat = P_hat Q^T; one warp per row, lanes over the columns.
// ---------------------------------------------------------------------------
template <int R, bool VEC>
__global__ void __launch_bounds__(kPsgdThreads)
    psgd_reconstruct_kernel(const __grid_constant__ PsgdArgs a) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int kWarps = kPsgdThreads / 32;
    for (long long t = blockIdx.x; t < a.tile0[a.count]; t += gridDim.x) {
        const int l = matrix_of(a, t);
        const int i = (int)(t - a.tile0[l]) * kWarps + warp;
        const int n = a.rows[l], m = a.cols[l];
        if (i >= n) continue;
        float p[R];
#pragma unroll
        for (int k = 0; k < R; ++k) p[k] = __ldg(a.p + a.poff[l] + (long long)i * R + k);
        const float* qm = a.q + a.qoff[l];
        float* out = a.out + a.goff[l] + (long long)i * m;
        if (VEC) {
            for (int j4 = lane; j4 < (m >> 2); j4 += 32) {
                float q[4 * R];
                const float4* q4 = reinterpret_cast<const float4*>(qm + (long long)j4 * 4 * R);
#pragma unroll
                for (int k = 0; k < R; ++k) {
                    const float4 v = __ldg(q4 + k);
                    q[4 * k] = v.x;
                    q[4 * k + 1] = v.y;
                    q[4 * k + 2] = v.z;
                    q[4 * k + 3] = v.w;
                }
                __stcs(reinterpret_cast<float4*>(out) + j4,
                       make_float4(lowrank_value<R>(p, q), lowrank_value<R>(p, q + R),
                                   lowrank_value<R>(p, q + 2 * R), lowrank_value<R>(p, q + 3 * R)));
            }
        } else {
            for (int j = lane; j < m; j += 32) out[j] = lowrank_value<R>(p, qm + (long long)j * R);
        }
    }
}

// ---------------------------------------------------------------------------
// reconstruct, every m a multiple of 4: tiles of (matrix, 1024 columns, 128
// rows).  A thread keeps the Q rows of its 4 columns in registers and runs
// down the tile's rows, whose P_hat rows are staged in shared memory; each
// row is one coalesced 16-byte store per thread.  Same fma chain as above.
// ---------------------------------------------------------------------------
constexpr int kRecRows = 128;

template <int R>
__global__ void __launch_bounds__(kPsgdThreads)
    psgd_reconstruct_cols_kernel(const __grid_constant__ PsgdArgs a) {
    constexpr int RP = Padded<R>::value;
    __shared__ __align__(16) float ps[kRecRows * RP];
    for (long long t = blockIdx.x; t < a.tile0[a.count]; t += gridDim.x) {
        const int l = matrix_of(a, t);
        const long long lt = t - a.tile0[l];
        const int n = a.rows[l], m = a.cols[l];
        const int rtiles = (n + kRecRows - 1) / kRecRows;
        const int ct = (int)(lt / rtiles);
        const int r0 = (int)(lt - (long long)ct * rtiles) * kRecRows;
        const int r1 = min(n, r0 + kRecRows);
        __syncthreads();  // the previous tile's reads of ps are done
        for (int x = threadIdx.x; x < (r1 - r0) * RP; x += kPsgdThreads) {
            const int i = x / RP, k = x - i * RP;
            ps[x] = k < R ? __ldg(a.p + a.poff[l] + (long long)(r0 + i) * R + k) : 0.f;
        }
        __syncthreads();
        const int j = ct * kBackColsPerTile + 4 * threadIdx.x;
        if (j >= m) continue;
        float q[4 * R];
        const float4* q4 = reinterpret_cast<const float4*>(a.q + a.qoff[l] + (long long)j * R);
#pragma unroll
        for (int k = 0; k < R; ++k) {
            const float4 v = __ldg(q4 + k);
            q[4 * k] = v.x;
            q[4 * k + 1] = v.y;
            q[4 * k + 2] = v.z;
            q[4 * k + 3] = v.w;
        }
        float* out = a.out + a.goff[l] + (long long)r0 * m + j;
        for (int i = 0; i < r1 - r0; ++i) {
            float p[R];
            const float* pr = ps + i * RP;
#pragma unroll
            for (int k = 0; k < R; ++k) p[k] = pr[k];
            __stcs(reinterpret_cast<float4*>(out + (long long)i * m),
                   make_float4(lowrank_value<R>(p, q), lowrank_value<R>(p, q + R),
                               lowrank_value<R>(p, q + 2 * R), lowrank_value<R>(p, q + 3 * R)));
        }
    }
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
static int grid_for(long long tiles, int sms, int per_sm) {
    const long long cap = (long long)sms * per_sm;
    const long long g = tiles < cap ? tiles : cap;
    return g < 1 ? 1 : (int)g;
}

// One resident wave of the kernel (grid-stride over its tiles).
static int resident_grid(const void* fn, size_t smem, long long tiles, int sms) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kPsgdThreads, smem) !=
            cudaSuccess ||
        per_sm < 1)
        per_sm = 1;
    return grid_for(tiles, sms, per_sm);
}

#define GQ_PSGD_RANKS(X) X(1) X(2) X(3) X(4) X(5) X(6) X(7) X(8)

template <int R, bool HP>
static cudaError_t project_inst(const PsgdArgs& a, int sms, cudaStream_t st) {
    auto kern = psgd_project_kernel<R, HP>;
    kern<<<resident_grid((const void*)kern, 0, a.tile0[a.count], sms), kPsgdThreads, 0, st>>>(a);
    return cudaGetLastError();
}

template <int R, bool HP>
static cudaError_t project_q_inst(const PsgdArgs& a, int sms, cudaStream_t st) {
    auto kern = psgd_project_q_kernel<R, HP>;
    const size_t smem = (size_t)kQStages * (32 * R + 8 * 4 * 32) * sizeof(float4);
    static int limits[64] = {};
    const cudaError_t e = ensure_dynamic_smem((const void*)kern, smem, limits);
    if (e != cudaSuccess) return e;
    kern<<<resident_grid((const void*)kern, smem, a.tile0[a.count], sms), kPsgdThreads, smem,
           st>>>(a);
    return cudaGetLastError();
}


cudaError_t launch_psgd_project(const PsgdArgs& a, bool vec, int sms, cudaStream_t st) {
    const bool hp = a.have_prev != 0;
    if (vec) {
        switch (a.rank) {
            case 1: return hp ? project_q_inst<1, true>(a, sms, st) : project_q_inst<1, false>(a, sms, st);
            case 2: return hp ? project_q_inst<2, true>(a, sms, st) : project_q_inst<2, false>(a, sms, st);
            case 3: return hp ? project_q_inst<3, true>(a, sms, st) : project_q_inst<3, false>(a, sms, st);
            case 4: return hp ? project_q_inst<4, true>(a, sms, st) : project_q_inst<4, false>(a, sms, st);
            case 5: return hp ? project_q_inst<5, true>(a, sms, st) : project_q_inst<5, false>(a, sms, st);
            case 6: return hp ? project_q_inst<6, true>(a, sms, st) : project_q_inst<6, false>(a, sms, st);
            case 7: return hp ? project_q_inst<7, true>(a, sms, st) : project_q_inst<7, false>(a, sms, st);
            default: return hp ? project_q_inst<8, true>(a, sms, st) : project_q_inst<8, false>(a, sms, st);
        }
    }
#define GQ_PROJ(RR) \
    case RR: return hp ? project_inst<RR, true>(a, sms, st) : project_inst<RR, false>(a, sms, st);
    switch (a.rank) {
        GQ_PSGD_RANKS(GQ_PROJ)
        default: return cudaErrorInvalidValue;
    }
#undef GQ_PROJ
}

cudaError_t launch_psgd_orth(const PsgdArgs& a, cudaStream_t st) {
#define GQ_ORTH(RR) \
    case RR: psgd_orth_kernel<RR><<<a.count, 1024, 0, st>>>(a); break;
    switch (a.rank) {
        GQ_PSGD_RANKS(GQ_ORTH)
        default: return cudaErrorInvalidValue;
    }
#undef GQ_ORTH
    return cudaGetLastError();
}

size_t psgd_back_smem(int rank, int chunk_rows, bool vec) {
    return (size_t)chunk_rows * (size_t)((rank + 3) & ~3) * sizeof(float) +
           (vec ? (size_t)kBackStages * kPsgdThreads * sizeof(float4) : 0);
}

template <int R, bool VEC>
static cudaError_t back_inst(const PsgdArgs& a, int sms, cudaStream_t st) {
    auto kern = psgd_back_kernel<R, VEC>;
    const size_t smem = psgd_back_smem(R, a.chunk_rows, VEC);
    static int limits[64] = {};
    const cudaError_t e = ensure_dynamic_smem((const void*)kern, smem, limits);
    if (e != cudaSuccess) return e;
    kern<<<resident_grid((const void*)kern, smem, a.tile0[a.count], sms), kPsgdThreads, smem,
           st>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_psgd_back(const PsgdArgs& a, bool vec, int sms, cudaStream_t st) {
#define GQ_BACK(RR) \
    case RR: return vec ? back_inst<RR, true>(a, sms, st) : back_inst<RR, false>(a, sms, st);
    switch (a.rank) {
        GQ_PSGD_RANKS(GQ_BACK)
        default: return cudaErrorInvalidValue;
    }
#undef GQ_BACK
}

cudaError_t launch_psgd_back_reduce(const PsgdArgs& a, int sms, cudaStream_t st) {
    psgd_back_reduce_kernel<<<grid_for(a.tile0[a.count], sms, 8), kPsgdThreads, 0, st>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_psgd_mean(const float* qsum, float* q, long long len, int W, int sms,
                             cudaStream_t st) {
    const long long blocks = (len + 255) / 256;
    psgd_mean_kernel<<<grid_for(blocks, sms, 8), 256, 0, st>>>(qsum, q, len, (float)W);
    return cudaGetLastError();
}

cudaError_t launch_psgd_reconstruct_cols(const PsgdArgs& a, int sms, cudaStream_t st) {
#define GQ_RECC(RR)                                                                    \
    case RR: {                                                                         \
        auto kern = psgd_reconstruct_cols_kernel<RR>;                                  \
        kern<<<resident_grid((const void*)kern, 0, a.tile0[a.count], sms), kPsgdThreads, 0, \
               st>>>(a);                                                               \
        break;                                                                         \
    }
    switch (a.rank) {
        GQ_PSGD_RANKS(GQ_RECC)
        default: return cudaErrorInvalidValue;
    }
#undef GQ_RECC
    return cudaGetLastError();
}

cudaError_t launch_psgd_reconstruct(const PsgdArgs& a, bool vec, int sms, cudaStream_t st) {
    const int grid = grid_for(a.tile0[a.count], sms, 8);
#define GQ_REC(RR)                                                                         \
    case RR:                                                                               \
        if (vec) psgd_reconstruct_kernel<RR, true><<<grid, kPsgdThreads, 0, st>>>(a);      \
        else psgd_reconstruct_kernel<RR, false><<<grid, kPsgdThreads, 0, st>>>(a);         \
        break;
    switch (a.rank) {
        GQ_PSGD_RANKS(GQ_REC)
        default: return cudaErrorInvalidValue;
    }
#undef GQ_REC
    return cudaGetLastError();
}

}  // namespace gq
