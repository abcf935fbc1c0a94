// gq_device.cuh -- device building blocks of libgq (sm_100a).
//
// Philox-4x32-10 in registers, the stochastic-rounding quantizers, and the
// warp-level packing of codes at wire width.  Every floating-point step that
// decides a code or an output uses an explicit _rn/_rd intrinsic, so the
// compiler can neither contract nor reorder it.
#pragma once

#include <cuda_fp16.h>

#include <cstdint>

namespace gq {

constexpr unsigned kFull = 0xFFFFFFFFu;

// ---------------------------------------------------------------------------
// Philox-4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As
// Easy as 1, 2, 3", SC'11): ten rounds of two 32x32->64 multiplies whose high
// halves are XORed with the other two counter words and the round key.  The
// round keys (key + r * Weyl constants) are the same for every thread, so the
// host computes them once and passes them in the kernel parameters.
// ---------------------------------------------------------------------------
struct RoundKeys {
    uint32_t k[20];  // k[2r], k[2r+1]: key words of round r
};

__device__ __forceinline__ uint4 philox10(uint4 c, const RoundKeys& rk) {
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        const unsigned long long p0 = (unsigned long long)c.x * 0xD2511F53ull;
        const unsigned long long p1 = (unsigned long long)c.z * 0xCD9E8D57ull;
        const uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        const uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        c = make_uint4(hi1 ^ c.y ^ rk.k[2 * r], lo1, hi0 ^ c.w ^ rk.k[2 * r + 1], lo0);
    }
    return c;
}

// Counter of the block that serves coordinates 4q..4q+3 of `worker` at `step`.
__device__ __forceinline__ uint4 philox_counter(unsigned long long q, uint32_t step,
                                                uint32_t worker) {
    return make_uint4((uint32_t)q, step, worker, (uint32_t)(q >> 32));
}

// philox10 on the counter (lo32 q, step, worker, hi32 q) with its first two
// rounds split by what they depend on.  Round 0 multiplies lo32 q (one product
// per coordinate block) and the worker word (one per worker and step).  Round
// 1 multiplies the word that came from the worker product and the step (one
// per worker) and the word that came from q (one per block).  Two XORs per
// (worker, block) join the halves.
struct PhiloxWorkerPart {
    uint32_t bx;  // round-1 word x before the block half: lo(worker*M1) ^ k2
    uint32_t hz;  // round-1 word z before the block half: hi(A*M0) ^ k3
    uint32_t lw;  // round-1 word w: lo(A*M0), A = hi(worker*M1) ^ step ^ k0
};
struct PhiloxBlockPart {
    uint32_t hx;  // hi(X*M1), X = hi(lo32q*M0) ^ hi32q ^ k1
    uint32_t lx;  // round-1 word y: lo(X*M1)
    uint32_t y;   // lo(lo32q*M0), joined into round-1 word z
};

__device__ __forceinline__ PhiloxWorkerPart philox_worker_part(uint32_t step, uint32_t worker,
                                                               const RoundKeys& rk) {
    const unsigned long long p1 = (unsigned long long)worker * 0xCD9E8D57ull;
    const uint32_t A = (uint32_t)(p1 >> 32) ^ step ^ rk.k[0];
    const unsigned long long p0 = (unsigned long long)A * 0xD2511F53ull;
    return PhiloxWorkerPart{(uint32_t)p1 ^ rk.k[2], (uint32_t)(p0 >> 32) ^ rk.k[3], (uint32_t)p0};
}

__device__ __forceinline__ PhiloxBlockPart philox_block_part(unsigned long long q,
                                                             const RoundKeys& rk) {
    const unsigned long long p0 = (unsigned long long)(uint32_t)q * 0xD2511F53ull;
    const uint32_t X = (uint32_t)(p0 >> 32) ^ (uint32_t)(q >> 32) ^ rk.k[1];
    const unsigned long long p1 = (unsigned long long)X * 0xCD9E8D57ull;
    return PhiloxBlockPart{(uint32_t)(p1 >> 32), (uint32_t)p1, (uint32_t)p0};
}

// philox10(philox_counter(q, step, worker), rk) from the two halves.
__device__ __forceinline__ uint4 philox10_split(const PhiloxBlockPart& b,
                                                const PhiloxWorkerPart& w,
                                                const RoundKeys& rk) {
    uint4 c = make_uint4(b.hx ^ w.bx, b.lx, b.y ^ w.hz, w.lw);
#pragma unroll
    for (int r = 2; r < 10; ++r) {
        const unsigned long long p0 = (unsigned long long)c.x * 0xD2511F53ull;
        const unsigned long long p1 = (unsigned long long)c.z * 0xCD9E8D57ull;
        const uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        const uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        c = make_uint4(hi1 ^ c.y ^ rk.k[2 * r], lo1, hi0 ^ c.w ^ rk.k[2 * r + 1], lo0);
    }
    return c;
}

// ---------------------------------------------------------------------------
// Stochastic rounding.  A magnitude y >= 0 becomes floor(y + u) with
// u = f * 2^-23, f the top 23 bits of a Philox word: that is floor(y) + 1
// exactly when frac(y) + u >= 1, an event of probability frac(y), so the
// rounding is unbiased.
//
// floor(y + u) is computed without a conversion instruction: U = 1 + u is
// built from bits (exact), t1 = fl_down(y + U) has the same floor as y + U
// (that floor is an integer <= 2^24, hence a float, and rounding down cannot
// cross it), and fl_down(t1 + 2^23) is 2^23 + floor(t1) exactly because floats
// in [2^23, 2^24) are the integers.  So the integer is the bit pattern minus
// that of 2^23, minus 1 for the U offset.  Valid for 0 <= y < 2^23 - 2.
// ---------------------------------------------------------------------------
// f = word >> 9 as the high half of word * 2^23, so that it runs on the
// multiply pipe (the logic pipe is the busier one in the fused pass).
__device__ __forceinline__ uint32_t top23(uint32_t word) {
    uint32_t r;
    asm("mul.hi.u32 %0, %1, %2;" : "=r"(r) : "r"(word), "r"(0x00800000u));
    return r;
}

// U = 1 + u as a float: exponent of 1.0 with f in the mantissa (the add is
// exact: f < 2^23 never reaches the exponent field).
__device__ __forceinline__ float unit_plus_u(uint32_t word) {
    uint32_t r;
    asm("mad.hi.u32 %0, %1, %2, %3;" : "=r"(r) : "r"(word), "r"(0x00800000u), "r"(0x3F800000u));
    return __uint_as_float(r);
}

__device__ __forceinline__ int floor_y_plus_u(float y, float U) {
    const float t1 = __fadd_rd(y, U);
    const float t2 = __fadd_rd(t1, 8388608.0f);
    return __float_as_int(t2) - 0x4B000001;
}

// Apply the sign of v (its sign bit, so -0.0 and +0.0 both give +k / -k = 0).
__device__ __forceinline__ int with_sign_of(int k, float v) {
    const int sgn = __float_as_int(v) >> 31;  // 0 or -1
    return (k ^ sgn) - sgn;
}

// Uniform levels {0, +-1/s, ..., +-1}: a = s/S rounded down, r = fl(v a) clamped to
// [-s, s] (fminf also maps a NaN product to s), code = floor(r + u).  The
// signed value is rounded directly: each coordinate gets the same two
// outcomes with the same probabilities as sign(v) * floor(|r| + u), and no
// sign handling is needed.  Same conversion-free floor as above, with base
// 1.5 * 2^23 so that negative sums stay in [2^23, 2^24).
__device__ __forceinline__ int quant_uniform(float v, float a, float smax, uint32_t word) {
    const float r = fmaxf(fminf(__fmul_rn(v, a), smax), -smax);
    const float t1 = __fadd_rd(r, unit_plus_u(word));
    const float t2 = __fadd_rd(t1, 12582912.0f);
    return __float_as_int(t2) - 0x4B400001;
}

// The same rounding, returned "biased": the float 1.5 * 2^23 + code, whose bit
// pattern is kCodeBias + code.  Adding 1.5 * 2^23 - 1 instead of 1.5 * 2^23
// absorbs the -1 of the U offset, so no per-element subtraction is needed: the
// low 8 / 16 bits of the pattern are already the int8 / int16 code, sums of
// patterns differ from sums of codes by a multiple of kCodeBias, and
// (pattern as float) - 1.5 * 2^23 is the code as a float, exactly.
constexpr uint32_t kCodeBias = 0x4B400000u;
__device__ __forceinline__ float quant_uniform_biased(float v, float a, float smax, uint32_t word) {
    const float r = fmaxf(fminf(__fmul_rn(v, a), smax), -smax);
    const float t1 = __fadd_rd(r, unit_plus_u(word));
    return __fadd_rd(t1, 12582911.0f);
}

// Without the clamp, for a scale S that bounds every input (|v| <= S, which
// gq_global_norm guarantees) and a = s/S rounded down: then |v a| <= s
// exactly, so |fl(v a)| <= s and the clamp could never act.
__device__ __forceinline__ float quant_uniform_biased_unclamped(float v, float a, uint32_t word) {
    const float t1 = __fadd_rd(__fmul_rn(v, a), unit_plus_u(word));
    return __fadd_rd(t1, 12582911.0f);
}

// Exponential levels {0, 2^-(L-1), ..., 1/2, 1}: a = fl(1/S), r = min(fl(|v| a), 1).
// For r >= 2^-(L-1), r = (1 + m 2^-23) 2^E with m the mantissa field: the
// bracket is [2^E, 2^(E+1)], the lower level has index L + E, and the
// round-up probability (r - 2^E)/2^E equals m 2^-23, so the decision
// frac + u >= 1 is the integer test m + f >= 2^23.  Below 2^-(L-1) the bracket
// is [0, 2^-(L-1)] and p = r 2^(L-1) (exact); p + u >= 1 iff fl_down(p + U) >= 2.
__device__ __forceinline__ int quant_exp(float v, float a, int L, float finest, float inv_finest,
                                         uint32_t word) {
    const float r = fminf(__fmul_rn(fabsf(v), a), 1.0f);
    const uint32_t f = top23(word);
    int idx;
    if (r >= finest) {
        const uint32_t rb = __float_as_uint(r);
        const int E = (int)(rb >> 23) - 127;
        idx = L + E + (int)(((rb & 0x007FFFFFu) + f) >> 23);
    } else {
        const float p = __fmul_rn(r, inv_finest);
        idx = __fadd_rd(p, __uint_as_float(0x3F800000u | f)) >= 2.0f ? 1 : 0;
    }
    return with_sign_of(idx, v);
}

// Exponential levels by the exponent carry, with the finest level moved onto
// 2^-126 so that no bracket needs a case of its own.  r = fl(v a) is scaled
// by shift = 2^(L-127) rounding toward zero: exact for |r| >= 2^-(L-1), and
// below that the subnormal result's mantissa is floor(p 2^23) with
// p = |r| 2^(L-1), the bottom bracket's round-up probability.  The 23 random
// bits f are added to the bit pattern in one multiply-add (the high half of
// word * 2^23 is word >> 9): the carry out of the mantissa is the round-up
// event m + f >= 2^23 in every bracket.  Masking the result to sign and
// exponent gives the rounded level +-2^(idx-127) (idx = the level index,
// exponent field 0 for the zero level); its top nine bits are sign and index.
__device__ __forceinline__ uint32_t exp_round_bits(float v, float a, float shift, uint32_t word) {
    const float rs = __fmul_rz(__fmul_rn(v, a), shift);
    uint32_t y;
    asm("mad.hi.u32 %0, %1, %2, %3;"
        : "=r"(y)
        : "r"(word), "r"(0x00800000u), "r"(__float_as_uint(rs)));
    return y;
}

// A float holding a sum of rounded levels from exp_round_bits, as the integer
// number of finest levels it holds: t = f 2^126 is that integer (exact), and
// for |t| < 2^22 the bits of 1.5 * 2^23 + t are those of 1.5 * 2^23 plus t.
__device__ __forceinline__ int float_units_to_int(float f) {
    const float t = __fmul_rn(f, 0x1p126f);
    return __float_as_int(__fadd_rn(t, 12582912.0f)) - 0x4B400000;
}

// Value a code adds to the sum: the code itself (uniform levels) or
// sign * 2^(idx-1) units of the finest level (exponential levels).
template <int LEVELS>
__device__ __forceinline__ int code_value(int code) {
    if (LEVELS == 0) return code;
    const int sgn = code >> 31;
    const int idx = (code ^ sgn) - sgn;
    const int mag = (1 << idx) >> 1;
    return (mag ^ sgn) - sgn;
}

// Exact int -> float for |x| < 2^22: 1.5 * 2^23 + x lies in [2^23, 2^24), where
// floats are the integers, so building it from bits and subtracting is exact.
__device__ __forceinline__ float small_int_to_float(int x) {
    return __fsub_rn(__int_as_float(0x4B400000 + x), 12582912.0f);
}

// ---------------------------------------------------------------------------
// Warp packing.  A warp covers one 128-coordinate block of one worker's row;
// lane l holds codes 4l..4l+3.  Wire layout: bits 4/5 -- little-endian
// bitstream of excess-2^(b-1) fields (code j at stream bits [b j, b j + b));
// 8 -- int8; 16 -- int16.  One block is 16 * BITS bytes, so every warp store
// is aligned and in range.
// ---------------------------------------------------------------------------

// PTX shifts clamp the amount to the register width (shift by >= 32 gives 0),
// unlike C++ shifts, so a lane can OR in a neighbour's chunk unconditionally.
__device__ __forceinline__ uint32_t shl_clamped(uint32_t x, uint32_t n) {
    uint32_t r;
    asm("shl.b32 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(n));
    return r;
}
__device__ __forceinline__ uint32_t shr_clamped(uint32_t x, uint32_t n) {
    uint32_t r;
    asm("shr.b32 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(n));
    return r;
}

template <int BITS>
struct Packer {
    // bits 5: lane k < 20 stores word k = stream bits [32k, 32k + 32), which
    // start inside the 20-bit chunk of lane src0 = floor(8k/5) at bit offset
    // off = 32k - 20 src0 and reach at most two chunks further.  Only lane 19
    // has src0 + 2 = 32; it reads lane 31 twice and its shift of 40 - off = 32
    // clears the second copy.
    int src0, src2;
    uint32_t sh0, sh1, sh2;
    __device__ __forceinline__ void init(int lane) {
        if (BITS == 5) {
            src0 = min((8 * lane) / 5, 30);
            src2 = min(src0 + 2, 31);
            const int off = lane < 20 ? 32 * lane - 20 * src0 : 0;  // lanes >= 20 store nothing
            sh0 = (uint32_t)off;
            sh1 = (uint32_t)(20 - off);
            sh2 = (uint32_t)(40 - off);
        }
    }
    // Pack and store the 4 codes of this lane; dst is the block's first byte.
    // The inputs are code + BIAS (mod 2^32) for a BIAS whose low 16 bits are
    // zero: the excess-field constants absorb it, and the int8 / int16 fields
    // are the low bits, which BIAS leaves untouched.
    template <uint32_t BIAS = 0u>
    __device__ __forceinline__ void store(int lane, int c0, int c1, int c2, int c3,
                                          unsigned char* dst) const {
        static_assert((BIAS & 0xFFFFu) == 0u, "bias must keep the low 16 bits");
        if (BITS == 5) {
            // excess-16 fields without masking: sum of c_i 32^i plus 16 * (1 + 32 + 1024 + 32768)
            constexpr uint32_t k5 = 541200u - BIAS * 33825u;
            const uint32_t x = (uint32_t)c0 + (uint32_t)c1 * 32u + (uint32_t)c2 * 1024u +
                               (uint32_t)c3 * 32768u + k5;
            const uint32_t x0 = __shfl_sync(kFull, x, src0);
            const uint32_t x1 = __shfl_sync(kFull, x, src0 + 1);
            const uint32_t x2 = __shfl_sync(kFull, x, src2);
            const uint32_t word = shr_clamped(x0, sh0) | shl_clamped(x1, sh1) | shl_clamped(x2, sh2);
            if (lane < 20) reinterpret_cast<uint32_t*>(dst)[lane] = word;
        } else if (BITS == 4) {
            // excess-8 fields: sum of c_i 16^i plus 8 * (1 + 16 + 256 + 4096)
            constexpr uint32_t k4 = 34952u - BIAS * 4369u;
            const uint32_t x = (uint32_t)c0 + (uint32_t)c1 * 16u + (uint32_t)c2 * 256u +
                               (uint32_t)c3 * 4096u + k4;
            const uint32_t xa = __shfl_sync(kFull, x, (2 * lane) & 31);
            const uint32_t xb = __shfl_sync(kFull, x, (2 * lane + 1) & 31);
            if (lane < 16) reinterpret_cast<uint32_t*>(dst)[lane] = xa | (xb << 16);
        } else if (BITS == 8) {
            const uint32_t x = (uint32_t)(c0 & 255) | ((uint32_t)(c1 & 255) << 8) |
                               ((uint32_t)(c2 & 255) << 16) | ((uint32_t)(c3 & 255) << 24);
            reinterpret_cast<uint32_t*>(dst)[lane] = x;
        } else if (BITS == 16) {
            uint2 x;
            x.x = (uint32_t)(c0 & 0xFFFF) | ((uint32_t)c1 << 16);
            x.y = (uint32_t)(c2 & 0xFFFF) | ((uint32_t)c3 << 16);
            reinterpret_cast<uint2*>(dst)[lane] = x;
        }
    }
};

// Unpacking: the inverse, reading one block of one worker's row.
template <int BITS>
struct Unpacker {
    int w0;   // bits 5: first word holding this lane's chunk
    int off;  // bits 5: bit offset of the chunk in that word
    __device__ __forceinline__ void init(int lane) {
        if (BITS == 5) {
            w0 = (20 * lane) >> 5;
            off = (20 * lane) & 31;
        }
    }
    __device__ __forceinline__ static int sext(uint32_t field, int bits) {
        return ((int)(field << (32 - bits))) >> (32 - bits);
    }
    __device__ __forceinline__ void load(int lane, const unsigned char* src, int& c0, int& c1,
                                         int& c2, int& c3) const {
        if (BITS == 5) {
            const uint32_t mine = lane < 20 ? reinterpret_cast<const uint32_t*>(src)[lane] : 0u;
            const uint32_t a = __shfl_sync(kFull, mine, w0);
            const uint32_t b = __shfl_sync(kFull, mine, min(w0 + 1, 31));
            const uint32_t x = __funnelshift_r(a, b, off);
            c0 = (int)(x & 31) - 16;
            c1 = (int)((x >> 5) & 31) - 16;
            c2 = (int)((x >> 10) & 31) - 16;
            c3 = (int)((x >> 15) & 31) - 16;
        } else if (BITS == 4) {
            const uint32_t mine = lane < 16 ? reinterpret_cast<const uint32_t*>(src)[lane] : 0u;
            const uint32_t wv = __shfl_sync(kFull, mine, lane >> 1);
            const uint32_t x = (lane & 1) ? (wv >> 16) : wv;
            c0 = (int)(x & 15) - 8;
            c1 = (int)((x >> 4) & 15) - 8;
            c2 = (int)((x >> 8) & 15) - 8;
            c3 = (int)((x >> 12) & 15) - 8;
        } else if (BITS == 8) {
            const uint32_t x = reinterpret_cast<const uint32_t*>(src)[lane];
            c0 = sext(x, 8);
            c1 = sext(x >> 8, 8);
            c2 = sext(x >> 16, 8);
            c3 = sext(x >> 24, 8);
        } else {
            const uint2 x = reinterpret_cast<const uint2*>(src)[lane];
            c0 = sext(x.x, 16);
            c1 = sext(x.x >> 16, 16);
            c2 = sext(x.y, 16);
            c3 = sext(x.y >> 16, 16);
        }
    }
};

// ---------------------------------------------------------------------------
// Per-coordinate outputs shared by the fused kernels.
// ---------------------------------------------------------------------------
// The [d] mean output: its base is 16-byte aligned and j0 % 4 == 0.  FULL:
// the caller knows that j0 + 3 < d.
template <bool FULL = false>
__device__ __forceinline__ void store_out4(float* out, long long j0, long long d, float4 v) {
    if (FULL || j0 + 3 < d) {
        __stcs(reinterpret_cast<float4*>(out + j0), v);
        return;
    }
    if (j0 < d) out[j0] = v.x;
    if (j0 + 1 < d) out[j0 + 1] = v.y;
    if (j0 + 2 < d) out[j0 + 2] = v.z;
}

__device__ __forceinline__ float4 add4(float4 a, float4 b) {
    return make_float4(__fadd_rn(a.x, b.x), __fadd_rn(a.y, b.y), __fadd_rn(a.z, b.z),
                       __fadd_rn(a.w, b.w));
}

// The fp16 wire type holds the integer sum itself: every integer of magnitude
// at most 2048 is an fp16 value, so int -> float -> fp16 and back are exact.
__device__ __forceinline__ uint32_t int_to_f16_bits(int x) {
    return (uint32_t)__half_as_ushort(__float2half_rn((float)x));
}
__device__ __forceinline__ int f16_bits_to_int(uint32_t h) {
    return (int)__half2float(__ushort_as_half((unsigned short)h));
}

// The [d] outputs (sum, mean) are vectors of their own: j0 is a multiple of 4,
// so a 4-wide store is aligned whenever all 4 coordinates are in range.
// wire: 1 int8, 2 int16, 3 fp16 holding the integer.
template <bool FULL = false>
__device__ __forceinline__ void store_sum_16(void* sum, long long j0, long long d, uint32_t s0,
                                             uint32_t s1, uint32_t s2, uint32_t s3) {
    unsigned short* p = reinterpret_cast<unsigned short*>(sum) + j0;
    if (FULL || j0 + 3 < d) {
        uint2 x;
        x.x = (s0 & 0xFFFFu) | (s1 << 16);
        x.y = (s2 & 0xFFFFu) | (s3 << 16);
        __stcs(reinterpret_cast<uint2*>(p), x);
    } else {
        if (j0 < d) p[0] = (unsigned short)s0;
        if (j0 + 1 < d) p[1] = (unsigned short)s1;
        if (j0 + 2 < d) p[2] = (unsigned short)s2;
    }
}

template <bool FULL = false>
__device__ __forceinline__ void store_sum(void* sum, int wire, long long j0, long long d, int s0,
                                          int s1, int s2, int s3) {
    if (wire == 3) {
        store_sum_16<FULL>(sum, j0, d, int_to_f16_bits(s0), int_to_f16_bits(s1),
                           int_to_f16_bits(s2), int_to_f16_bits(s3));
        return;
    }
    if (wire == 1) {
        signed char* p = reinterpret_cast<signed char*>(sum) + j0;
        if (FULL || j0 + 3 < d) {
            const uint32_t x = (uint32_t)(s0 & 255) | ((uint32_t)(s1 & 255) << 8) |
                               ((uint32_t)(s2 & 255) << 16) | ((uint32_t)(s3 & 255) << 24);
            __stcs(reinterpret_cast<unsigned int*>(p), x);
        } else {
            if (j0 < d) p[0] = (signed char)s0;
            if (j0 + 1 < d) p[1] = (signed char)s1;
            if (j0 + 2 < d) p[2] = (signed char)s2;
        }
    } else {
        store_sum_16<FULL>(sum, j0, d, (uint32_t)s0, (uint32_t)s1, (uint32_t)s2, (uint32_t)s3);
    }
}

__device__ __forceinline__ void load_sum(const void* sum, int wire, long long j0, long long d,
                                         int& s0, int& s1, int& s2, int& s3) {
    if (wire == 1) {
        const signed char* p = reinterpret_cast<const signed char*>(sum) + j0;
        if (j0 + 3 < d) {
            const uint32_t x = __ldcs(reinterpret_cast<const unsigned int*>(p));
            s0 = (int)(signed char)(x & 255);
            s1 = (int)(signed char)((x >> 8) & 255);
            s2 = (int)(signed char)((x >> 16) & 255);
            s3 = (int)(signed char)(x >> 24);
        } else {
            s0 = j0 < d ? p[0] : 0;
            s1 = j0 + 1 < d ? p[1] : 0;
            s2 = j0 + 2 < d ? p[2] : 0;
            s3 = 0;
        }
    } else {
        const short* p = reinterpret_cast<const short*>(sum) + j0;
        if (j0 + 3 < d) {
            const uint2 x = __ldcs(reinterpret_cast<const uint2*>(p));
            s0 = (int)(short)(x.x & 0xFFFF);
            s1 = (int)(short)(x.x >> 16);
            s2 = (int)(short)(x.y & 0xFFFF);
            s3 = (int)(short)(x.y >> 16);
        } else {
            s0 = j0 < d ? p[0] : 0;
            s1 = j0 + 1 < d ? p[1] : 0;
            s2 = j0 + 2 < d ? p[2] : 0;
            s3 = 0;
        }
        if (wire == 3) {
            s0 = f16_bits_to_int((uint32_t)s0 & 0xFFFFu);
            s1 = f16_bits_to_int((uint32_t)s1 & 0xFFFFu);
            s2 = f16_bits_to_int((uint32_t)s2 & 0xFFFFu);
            s3 = f16_bits_to_int((uint32_t)s3 & 0xFFFFu);
        }
    }
}

// Decoded mean of one summed integer: fl(fl(sum * c) / W).
__device__ __forceinline__ float decode_mean(int s, float c, float inv_w, int w_pow2, int W) {
    const float y = __fmul_rn(small_int_to_float(s), c);
    return w_pow2 ? __fmul_rn(y, inv_w) : __fdiv_rn(y, (float)W);
}

}  // namespace gq
