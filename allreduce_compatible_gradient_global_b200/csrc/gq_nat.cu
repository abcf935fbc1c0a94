// gq_nat.cu -- natural compression on the GPU (sm_100a).
//
// Horvath, Ho, Horvath, Sahu, Canini, Richtarik, "Natural Compression for
// Distributed Deep Learning" (MSML 2022), cited in the reference list of
// "Global-QSGD: Allreduce-Compatible Quantization for Distributed Learning with
// Theoretical Guarantees": every value is rounded stochastically to one of the
// two powers of two around it, unbiased, so that only its sign and exponent
// travel.
//
// In the binary32 pattern of x the rounding is one integer add: with f the
// top 23 bits of a Philox word, pattern + f carries out of the mantissa field
// exactly when m + f >= 2^23 (probability m 2^-23 = |x|/2^e - 1) and bumps the
// exponent to the upper power of two; the top nine bits of the sum are then
// the sign and exponent of the result.  A subnormal (exponent field 0) rounds
// between 0 and 2^-126 by the same carry.
//
// nat_quantize_kernel: one grid row per worker, one thread per group of four
// coordinates (on vector rows, kNatStages - 1 groups in flight per thread
// through a cp.async ring in shared memory); the
// group's Philox block serves its four coordinates (word k for coordinate
// 4q + k).  nat_decode_sum_kernel: one thread per group of four coordinates,
// fp32 sum over workers in ascending order.  Both stream HBM: 4 B read + 2 B
// written per worker-coordinate, then 2 B read per worker-coordinate + 4 B
// written per coordinate.
#include "gq_nat.h"

namespace gq {

namespace {

// The code of one value: sign << 8 | biased exponent of the rounded result.
// Inputs with exponent field 255 (inf, NaN) keep their own top nine bits.
__device__ __forceinline__ uint32_t nat_code(float x, uint32_t word, bool& bad) {
    const uint32_t u = __float_as_uint(x);
    const bool special = (u & 0x7F800000u) == 0x7F800000u;
    const uint32_t c = special ? (u >> 23) : ((u + top23(word)) >> 23);
    bad |= (c & 0xFFu) == 0xFFu;  // inf / NaN in, or a rounding past the largest float
    return c;
}

__device__ __forceinline__ float nat_value(uint32_t code) { return __uint_as_float(code << 23); }

// Vector rows: every thread streams its groups through a private ring of
// kNatStages 16-byte slots in shared memory, filled by cp.async, so that
// kNatStages - 1 loads stay in flight while Philox runs on the current group,
// without holding registers for them.  A thread reads back only its own slots
// after its own cp.async.wait_group, so no block barrier is needed.
constexpr int kNatStages = 8;

__device__ __forceinline__ void nat_cp_async16(void* smem_dst, const void* gmem_src) {
    const uint32_t d = (uint32_t)__cvta_generic_to_shared(smem_dst);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gmem_src) : "memory");
}

__device__ __forceinline__ void nat_cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}

template <int N>
__device__ __forceinline__ void nat_cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <bool VEC>
__global__ void __launch_bounds__(kThreads) nat_quantize_kernel(const __grid_constant__ NatArgs a) {
    const uint32_t step = a.step_dev ? __ldg(a.step_dev) : a.step;
    const int w = blockIdx.y;  // one grid row per worker
    const uint32_t wid = a.worker0 + (uint32_t)w;
    const long long nq = (a.n + 3) >> 2;
    const long long stride = (long long)gridDim.x * blockDim.x;
    const float* xr = a.x + (long long)w * a.n;
    unsigned short* cr = a.codes + (long long)w * a.n;
    bool bad = false;
    if (VEC) {  // n % 4 == 0: every group is whole and 16-byte aligned
        __shared__ float4 ring[kNatStages][kThreads];
        const long long q0 = (long long)blockIdx.x * blockDim.x + threadIdx.x;
        const long long nit = q0 < nq ? (nq - q0 + stride - 1) / stride : 0;
        const float4* x4 = reinterpret_cast<const float4*>(xr);
#pragma unroll
        for (int k = 0; k < kNatStages - 1; ++k) {
            if (k < nit) nat_cp_async16(&ring[k][threadIdx.x], x4 + q0 + k * stride);
            nat_cp_async_commit();
        }
        for (long long it = 0; it < nit; ++it) {
            const long long ahead = it + kNatStages - 1;
            if (ahead < nit)
                nat_cp_async16(&ring[ahead % kNatStages][threadIdx.x], x4 + q0 + ahead * stride);
            nat_cp_async_commit();
            nat_cp_async_wait<kNatStages - 1>();  // this thread's copy of group `it` landed
            const float4 v = ring[it % kNatStages][threadIdx.x];
            const long long q = q0 + it * stride;
            const uint4 rnd = philox10(philox_counter((unsigned long long)q, step, wid), a.rk);
            const uint32_t c0 = nat_code(v.x, rnd.x, bad), c1 = nat_code(v.y, rnd.y, bad);
            const uint32_t c2 = nat_code(v.z, rnd.z, bad), c3 = nat_code(v.w, rnd.w, bad);
            __stcs(reinterpret_cast<uint2*>(cr) + q, make_uint2(c0 | (c1 << 16), c2 | (c3 << 16)));
        }
        nat_cp_async_wait<0>();
    } else {
        for (long long q = (long long)blockIdx.x * blockDim.x + threadIdx.x; q < nq;
             q += stride) {
            const uint4 rnd = philox10(philox_counter((unsigned long long)q, step, wid), a.rk);
            const long long j0 = q << 2;
            const long long left = a.n - j0;
            const uint32_t words[4] = {rnd.x, rnd.y, rnd.z, rnd.w};
#pragma unroll
            for (int k = 0; k < 4; ++k)
                if (k < left)
                    cr[j0 + k] = (unsigned short)nat_code(__ldcs(xr + j0 + k), words[k], bad);
        }
    }
    if (bad) atomicOr(&a.hdr->flags, kFlagNonfiniteNat);
}

template <bool VEC>
__global__ void __launch_bounds__(kThreads)
    nat_decode_sum_kernel(const __grid_constant__ NatArgs a) {
    const long long nq = (a.n + 3) >> 2;
    for (long long q = (long long)blockIdx.x * blockDim.x + threadIdx.x; q < nq;
         q += (long long)gridDim.x * blockDim.x) {
        const long long j0 = q << 2;
        if (VEC) {
            // rows of 8-byte code groups; up to 8 workers' loads are issued
            // before the ordered sum consumes them
            const uint2* c = reinterpret_cast<const uint2*>(a.ccodes) + q;
            const long long row = a.n >> 2;
            uint2 p = __ldcs(c);
            float4 acc = make_float4(nat_value(p.x & 0xFFFFu), nat_value(p.x >> 16),
                                     nat_value(p.y & 0xFFFFu), nat_value(p.y >> 16));
            for (int w0 = 1; w0 < a.W; w0 += 8) {
                uint2 ps[8];
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    if (w0 + k < a.W) ps[k] = __ldcs(c + (long long)(w0 + k) * row);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    if (w0 + k < a.W) {
                        acc.x = __fadd_rn(acc.x, nat_value(ps[k].x & 0xFFFFu));
                        acc.y = __fadd_rn(acc.y, nat_value(ps[k].x >> 16));
                        acc.z = __fadd_rn(acc.z, nat_value(ps[k].y & 0xFFFFu));
                        acc.w = __fadd_rn(acc.w, nat_value(ps[k].y >> 16));
                    }
                }
            }
            __stcs(reinterpret_cast<float4*>(a.out + j0), acc);
        } else {
            const long long left = a.n - j0;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                if (k < left) {
                    float acc = nat_value(a.ccodes[j0 + k]);
                    for (int w = 1; w < a.W; ++w)
                        acc = __fadd_rn(acc, nat_value(a.ccodes[(long long)w * a.n + j0 + k]));
                    a.out[j0 + k] = acc;
                }
            }
        }
    }
}

int resident_blocks(const void* fn) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, kThreads, 0) != cudaSuccess || n < 1)
        n = 1;
    return n;
}

int grid_over(long long items, int sms, const void* fn) {
    const long long need = (items + kThreads - 1) / kThreads;
    const long long cap = (long long)sms * resident_blocks(fn);
    const long long g = need < cap ? need : cap;
    return g < 1 ? 1 : (int)g;
}

}  // namespace

// Grid (x, W): one row of blocks per worker, the resident wave split evenly
// between the rows (at least one block each).
cudaError_t launch_nat_quantize(const NatArgs& a, bool vec, int sms, cudaStream_t st) {
    const long long nq = (a.n + 3) >> 2;
    const void* fn = vec ? (const void*)nat_quantize_kernel<true>
                         : (const void*)nat_quantize_kernel<false>;
    const long long per_row = (long long)sms * resident_blocks(fn) / a.W;
    const long long need = (nq + kThreads - 1) / kThreads;
    long long gx = need < per_row ? need : per_row;
    if (gx < 1) gx = 1;
    const dim3 grid((unsigned)gx, (unsigned)a.W);
    if (vec)
        nat_quantize_kernel<true><<<grid, kThreads, 0, st>>>(a);
    else
        nat_quantize_kernel<false><<<grid, kThreads, 0, st>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_nat_decode_sum(const NatArgs& a, bool vec, int sms, cudaStream_t st) {
    const long long items = (a.n + 3) >> 2;
    if (vec) {
        const void* fn = (const void*)nat_decode_sum_kernel<true>;
        nat_decode_sum_kernel<true><<<grid_over(items, sms, fn), kThreads, 0, st>>>(a);
    } else {
        const void* fn = (const void*)nat_decode_sum_kernel<false>;
        nat_decode_sum_kernel<false><<<grid_over(items, sms, fn), kThreads, 0, st>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace gq
