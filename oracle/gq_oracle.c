/*
 * gq_oracle.c -- CPU oracle for allreduce-compatible global gradient
 * quantization.  TEST INFRASTRUCTURE ONLY (see gq_oracle.h): loaded by the
 * tests, the smoke check and the benchmark's CPU-baseline leg, never by the
 * product library.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -shared -fPIC.
 * All float arithmetic below is IEEE fp32 (SSE on x86-64, FLT_EVAL_METHOD 0)
 * unless a variable is declared double.
 */
#include "gq_oracle.h"

#include <math.h>
#include <stddef.h>
#include <string.h>

/* ------------------------------------------------------------------------
 * Philox-4x32-R.  Salmon et al., SC'11, section on the Philox family: each
 * round multiplies counter words 0 and 2 by two fixed odd constants, takes
 * the high and low 32-bit halves, XORs the high halves with the other two
 * counter words and the round key, and permutes; the key advances by a Weyl
 * sequence (golden ratio and sqrt(3)-1 fractions) between rounds.
 * ---------------------------------------------------------------------- */
void gqo_philox4x32(uint32_t ctr[4], uint32_t k0, uint32_t k1, int rounds)
{
    const uint32_t mult0 = 0xD2511F53u, mult1 = 0xCD9E8D57u;
    const uint32_t weyl0 = 0x9E3779B9u, weyl1 = 0xBB67AE85u;
    for (int r = 0; r < rounds; ++r) {
        if (r > 0) {
            k0 += weyl0;
            k1 += weyl1;
        }
        uint64_t prod0 = (uint64_t)mult0 * (uint64_t)ctr[0];
        uint64_t prod1 = (uint64_t)mult1 * (uint64_t)ctr[2];
        uint32_t n0 = (uint32_t)(prod1 >> 32) ^ ctr[1] ^ k0;
        uint32_t n1 = (uint32_t)prod1;
        uint32_t n2 = (uint32_t)(prod0 >> 32) ^ ctr[3] ^ k1;
        uint32_t n3 = (uint32_t)prod0;
        ctr[0] = n0;
        ctr[1] = n1;
        ctr[2] = n2;
        ctr[3] = n3;
    }
}

uint32_t gqo_uniform_bits(uint64_t seed, uint32_t tag, uint32_t step,
                          uint32_t worker, uint64_t j)
{
    uint64_t q = j >> 2;
    uint32_t ctr[4];
    ctr[0] = (uint32_t)q;
    ctr[1] = step;
    ctr[2] = worker;
    ctr[3] = (uint32_t)(q >> 32);
    gqo_philox4x32(ctr, (uint32_t)seed, (uint32_t)(seed >> 32) ^ tag, 10);
    return ctr[j & 3] >> 9; /* the top 23 bits */
}

/* Stochastic rounding decision shared by every quantizer here.
 * A magnitude y = l + p with integer l and fraction p in [0,1) rounds to
 * l + 1 exactly when p + u >= 1, u = f * 2^-23 uniform on [0,1); this happens
 * with probability p (up to the 2^-23 grid), so E[rounded] = y: the
 * unbiasedness that [GQ] and [SM] build on.  (p + u >= 1 is used rather than
 * u < p; both have probability p.)  The test is exact in double: p has 24
 * significant bits and u is a multiple of 2^-23, so whenever p >= 2^-30 the
 * sum is exact in 53 bits, and when p < 2^-30 the sum stays below
 * 1 - 2^-24 and no rounding reaches 1. */
static int round_up(float p, uint32_t f)
{
    double u = (double)f * (1.0 / 8388608.0);
    return ((double)p + u) >= 1.0;
}

static int sign_negative(float v)
{
    return signbit(v) != 0;
}

/* ------------------------------------------------------------------------
 * Global scale.  [GQ] Abstract: one norm-based scale shared by all workers.
 * The norm is the per-worker L2 norm and the shared value is the maximum
 * over workers (a reading: it is the smallest scale under which every
 * worker's |v_j|/S <= 1, the condition the level sets need).  [NUQ]
 * Abstract: QSGDinf scales by the max norm instead.
 * ---------------------------------------------------------------------- */
double gqo_sumsq(const float* g, const float* e, int64_t n)
{
    return gqo_sumsq_from(0.0, g, e, n);
}

double gqo_sumsq_from(double acc, const float* g, const float* e, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) {
        float v = e ? g[i] + e[i] : g[i];
        double dv = (double)v;
        acc = acc + dv * dv;
    }
    return acc;
}

float gqo_maxabs(const float* g, const float* e, int64_t n)
{
    float m = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float v = e ? g[i] + e[i] : g[i];
        float a = fabsf(v);
        if (isnan(a)) return a;
        if (a > m) m = a;
    }
    return m;
}

int gqo_global_scale(const float* g, const float* e, int W, int64_t d,
                     int scale_kind, float* S_out, double* norms_out)
{
    if (!g || W < 1 || d < 0 || !S_out) return -1;
    if (scale_kind != GQO_SCALE_L2 && scale_kind != GQO_SCALE_MAXABS) return -1;
    double best = 0.0;
    int saw_nan = 0;
    for (int w = 0; w < W; ++w) {
        const float* gw = g + (int64_t)w * d;
        const float* ew = e ? e + (int64_t)w * d : NULL;
        double n_w;
        if (scale_kind == GQO_SCALE_L2)
            n_w = sqrt(gqo_sumsq(gw, ew, d));
        else
            n_w = (double)gqo_maxabs(gw, ew, d);
        if (norms_out) norms_out[w] = n_w;
        if (isnan(n_w)) saw_nan = 1;
        else if (n_w > best) best = n_w;
    }
    *S_out = saw_nan ? NAN : (float)best;
    return 0;
}

/* ------------------------------------------------------------------------
 * Quantizers.
 *
 * UNIFORM ([NUQ] Abstract names QSGD; [GQ] gives the shared scale): levels
 * {0, +-1/s, ..., +-1} of S.  a = s/S rounded toward zero; r = fl(v*a)
 * (signed), clamped to [-s, s] (a guard: with |v| <= S it never acts);
 * l = floor(r), p = r - l
 * (exact, also for negative r); code = l + [p + u >= 1].  Rounding the signed
 * value this way gives each coordinate the same two outcomes with the same
 * probabilities as attaching v's sign to the rounded magnitude (for r = -2.3:
 * -3 with probability 0.3, -2 with probability 0.7), so the quantizer is the
 * same unbiased random variable; only the coupling to u differs.
 *
 * EXP ([NUQ] Abstract: nonuniform levels): levels {0, 2^-(L-1), ..., 1/2, 1}
 * of S.  a = 1/S rounded toward zero; r = fl(|v|*a), clamped to 1 (a guard:
 * with |v| <= S it never acts).  If r >= 2^-(L-1) write
 * r = f * 2^E with f in [1,2) (exponent read off the float, as frexp does):
 * the bracketing levels are 2^E and 2^(E+1), the lower one has index
 * L + E (index i stands for 2^(i-L)), and the round-up probability
 * (r - 2^E)/(2^(E+1) - 2^E) = f - 1 is exact.  Below 2^-(L-1) the bracket is
 * [0, 2^-(L-1)], index 0, and p = r * 2^(L-1) (exact).
 *
 * A scale that is zero or not finite gives a = 0, hence all codes 0.
 * ---------------------------------------------------------------------- */
/* a = the largest float with a * S <= s, i.e. s/S rounded toward zero.
 * Rounding down means |v| * a <= s exactly whenever |v| <= S, so no level
 * above s is ever reached for a scale that bounds the inputs (the clamp below
 * then never acts).  Found from the nearest float by stepping one ulp at a
 * time; a * S is exact in double (24 + 24 significant bits). */
static float uniform_magnitude_ratio(int s, float S)
{
    if (!(S > 0.0f) || !isfinite(S)) return 0.0f;
    double sd = (double)s;
    float a = (float)(sd / (double)S);
    while ((double)a * (double)S > sd) a = nextafterf(a, 0.0f);
    for (;;) {
        float up = nextafterf(a, INFINITY);
        if ((double)up * (double)S > sd) break;
        a = up;
    }
    return a;
}

float gqo_uniform_multiplier(int s, float S)
{
    return uniform_magnitude_ratio(s, S);
}

/* The same decision for a signed r = l + p, l = floor(r): round up exactly
 * when r + u >= l + 1, i.e. code = floor(r + u).  The fraction p = r - l of a
 * negative r is not always a float (r = -(u + 2^-26) with u in [1/8, 1/4) has
 * p = 1 - u - 2^-26, which a float subtraction rounds to 1 - u), so the
 * comparison is made on r + u itself, in double.  It is exact: r + u can
 * round only when r carries bits below 2^-38, i.e. |r| < 2^-14, and then
 * l + 1 is 0 or 1, which no such sum reaches by rounding. */
static int round_up_signed(float r, float l, uint32_t f)
{
    double u = (double)f * (1.0 / 8388608.0);
    return ((double)r + u) >= (double)l + 1.0;
}

static int32_t quantize_uniform(float v, float a, int s, uint32_t f)
{
    float r = v * a;
    float smax = (float)s;
    if (!(r <= smax)) r = smax; /* also maps NaN to s, as fminf does */
    if (r < -smax) r = -smax;
    float l = floorf(r);
    return (int32_t)l + round_up_signed(r, l, f);
}

static int32_t quantize_exp(float v, float a, int L, uint32_t f)
{
    float r = fabsf(v) * a;
    if (!(r <= 1.0f)) r = 1.0f;
    float finest = ldexpf(1.0f, -(L - 1));
    int32_t idx_lo;
    float p;
    if (r >= finest) {
        int e2;
        (void)frexpf(r, &e2); /* r = m * 2^e2 with m in [0.5, 1) */
        int E = e2 - 1;       /* so r = (2m) * 2^E with 2m in [1, 2) */
        float lower = ldexpf(1.0f, E);
        p = r / lower - 1.0f;
        idx_lo = L + E;
    } else {
        p = r * ldexpf(1.0f, L - 1);
        idx_lo = 0;
    }
    int32_t k = idx_lo + round_up(p, f);
    return sign_negative(v) ? -k : k;
}

int gqo_quantize(const float* g, const float* e, int W, int64_t n,
                 const int64_t* js, int levels, int s, int L,
                 uint64_t seed, uint32_t step, float S, int32_t* codes_out)
{
    return gqo_quantize_workers(g, e, W, n, js, 0u, levels, s, L, seed, step, S,
                                codes_out);
}

int gqo_quantize_workers(const float* g, const float* e, int W, int64_t n,
                         const int64_t* js, uint32_t worker0, int levels, int s,
                         int L, uint64_t seed, uint32_t step, float S,
                         int32_t* codes_out)
{
    if (!g || !codes_out || W < 1 || n < 0) return -1;
    if (levels == GQO_UNIFORM) {
        if (s < 1) return -1;
    } else if (levels == GQO_EXP) {
        if (L < 1 || L > 15) return -1;
    } else {
        return -1;
    }
    /* uniform: s/S, exponential: 1/S, both rounded toward zero */
    float a = uniform_magnitude_ratio(levels == GQO_UNIFORM ? s : 1, S);
    for (int w = 0; w < W; ++w) {
        for (int64_t i = 0; i < n; ++i) {
            int64_t at = (int64_t)w * n + i;
            float v = e ? g[at] + e[at] : g[at];
            uint64_t j = js ? (uint64_t)js[i] : (uint64_t)i;
            uint32_t f = gqo_uniform_bits(seed, 0u, step, worker0 + (uint32_t)w, j);
            codes_out[at] = (levels == GQO_UNIFORM)
                                ? quantize_uniform(v, a, s, f)
                                : quantize_exp(v, a, L, f);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------
 * Summation units.  [GQ][SM]: codes must be summable by Allreduce, i.e. the
 * decoded sum must equal the sum of the decoded codes.  Uniform codes are
 * already integer multiples of one step S/s.  Exponential level indices are
 * not additive, so each index is mapped to integer multiples of the finest
 * level before the sum: index i >= 1 -> 2^(i-1) units of 2^-(L-1).
 * ---------------------------------------------------------------------- */
int32_t gqo_code_value(int32_t code, int levels, int L)
{
    (void)L;
    if (levels == GQO_UNIFORM) return code;
    int32_t idx = code < 0 ? -code : code;
    int32_t mag = idx == 0 ? 0 : (int32_t)1 << (idx - 1);
    return code < 0 ? -mag : mag;
}

/* ------------------------------------------------------------------------
 * Wire packing (a reading: the pages fix only the bit count, [LQ] "Core
 * claim": b-bit indices are sent instead of 32-bit floats).  A row holds
 * ceil(d/128) blocks of 128 codes; coordinates past d carry code 0.
 *  bits 4, 5: little-endian bitstream, code j in stream bits [b*j, b*j + b),
 *             stored in excess-2^(b-1) form (field = code + 2^(b-1), so the
 *             codes -(2^(b-1)-1) .. 2^(b-1)-1 use fields 1 .. 2^b - 1);
 *  bits 8, 16: one two's-complement int8 / int16 per code.
 * ---------------------------------------------------------------------- */
int64_t gqo_packed_row_bytes(int bits, int64_t d)
{
    if (d < 0) return -1;
    if (bits != 4 && bits != 5 && bits != 8 && bits != 16) return -1;
    int64_t blocks = (d + 127) / 128;
    return blocks * 16 * bits;
}

static int32_t field_bias(int bits)
{
    return (bits == 4 || bits == 5) ? (int32_t)1 << (bits - 1) : 0;
}

int gqo_pack(const int32_t* codes, int W, int64_t d, int bits, uint8_t* out)
{
    int64_t rb = gqo_packed_row_bytes(bits, d);
    if (rb < 0 || !codes || !out || W < 1) return -1;
    int32_t hi = (1 << (bits - 1)) - 1;
    int32_t lo = (bits == 4 || bits == 5) ? -hi : -hi - 1;
    int64_t padded = rb * 8 / bits; /* codes per row, padding included */
    memset(out, 0, (size_t)(rb * W));
    for (int w = 0; w < W; ++w) {
        uint8_t* row = out + (int64_t)w * rb;
        for (int64_t j = 0; j < padded; ++j) {
            int32_t c = j < d ? codes[(int64_t)w * d + j] : 0;
            if (c < lo || c > hi) return -2;
            uint32_t field = (uint32_t)(c + field_bias(bits)) & ((1u << bits) - 1u);
            if (bits == 8) {
                row[j] = (uint8_t)field;
            } else if (bits == 16) {
                row[2 * j] = (uint8_t)(field & 0xFFu);
                row[2 * j + 1] = (uint8_t)(field >> 8);
            } else {
                /* bit by bit: bit t of the field goes to stream bit b*j + t,
                 * stream bit k lives in byte k/8 at position k%8 */
                for (int t = 0; t < bits; ++t) {
                    int64_t k = (int64_t)bits * j + t;
                    if ((field >> t) & 1u) row[k / 8] |= (uint8_t)(1u << (k % 8));
                }
            }
        }
    }
    return 0;
}

int gqo_unpack(const uint8_t* packed, int W, int64_t d, int bits,
               int32_t* codes_out)
{
    int64_t rb = gqo_packed_row_bytes(bits, d);
    if (rb < 0 || !packed || !codes_out || W < 1) return -1;
    for (int w = 0; w < W; ++w) {
        const uint8_t* row = packed + (int64_t)w * rb;
        for (int64_t j = 0; j < d; ++j) {
            uint32_t field = 0;
            if (bits == 8) {
                field = row[j];
            } else if (bits == 16) {
                field = (uint32_t)row[2 * j] | ((uint32_t)row[2 * j + 1] << 8);
            } else {
                for (int t = 0; t < bits; ++t) {
                    int64_t k = (int64_t)bits * j + t;
                    if ((row[k / 8] >> (k % 8)) & 1u) field |= 1u << t;
                }
            }
            int32_t c;
            if (bits == 4 || bits == 5) {
                c = (int32_t)field - field_bias(bits);
            } else {
                c = (int32_t)field;
                if (field & (1u << (bits - 1))) c -= (int32_t)1 << bits;
            }
            codes_out[(int64_t)w * d + j] = c;
        }
    }
    return 0;
}

int gqo_aggregate(const int32_t* codes, int W, int64_t n, int levels, int L,
                  int32_t* sum_out)
{
    if (!codes || !sum_out || W < 1 || n < 0) return -1;
    for (int64_t i = 0; i < n; ++i) {
        int32_t acc = 0;
        for (int w = 0; w < W; ++w)
            acc += gqo_code_value(codes[(int64_t)w * n + i], levels, L);
        sum_out[i] = acc;
    }
    return 0;
}

/* One step of value in the output units: S/s (UNIFORM) or S * 2^-(L-1). */
static float value_unit(int levels, int s, int L, float S)
{
    if (levels == GQO_UNIFORM) return S / (float)s;
    return S * ldexpf(1.0f, -(L - 1));
}

int gqo_decode_mean(const int32_t* sum, int64_t n, int W, int levels, int s,
                    int L, float S, float* out)
{
    if (!sum || !out || W < 1 || n < 0) return -1;
    if (levels == GQO_UNIFORM ? s < 1 : (L < 1 || L > 15)) return -1;
    float c = value_unit(levels, s, L, S);
    float fw = (float)W;
    for (int64_t i = 0; i < n; ++i) {
        float y = (float)sum[i] * c;
        out[i] = y / fw;
    }
    return 0;
}

/* Error feedback, [LQ] "What carries the argument": the residual of the
 * compression is kept and added to the next gradient. */
int gqo_error_feedback(const float* g, const float* e_in,
                       const int32_t* codes, int W, int64_t n, int levels,
                       int s, int L, float S, float* e_out)
{
    if (!g || !codes || !e_out || W < 1 || n < 0) return -1;
    if (levels == GQO_UNIFORM ? s < 1 : (L < 1 || L > 15)) return -1;
    float c = value_unit(levels, s, L, S);
    for (int64_t at = 0; at < (int64_t)W * n; ++at) {
        float v = e_in ? g[at] + e_in[at] : g[at];
        float q = (float)gqo_code_value(codes[at], levels, L) * c;
        e_out[at] = v - q;
    }
    return 0;
}

/* ------------------------------------------------------------------------
 * [LQ] log quantizer.  "Core claim": q(x) = sign(x) log(1 + a|x|)/log(1 + a)
 * on entries of each low-rank factor, then 2^b uniform bins, b = 8.
 * Referee major comment 1: the map is bounded only after normalising by the
 * maximum magnitude, so x/max|M| is used (per worker, per factor matrix).
 * Reading of the bins: sign + 127 magnitude steps of |q| in [0,1], so zero is
 * exact and the code is symmetric (255 of the 256 int8 values).  Rounding is
 * stochastic, as above.  Eq. (6) inverts the map: |x| = ((1+a)^|q| - 1)/a.
 * ---------------------------------------------------------------------- */
float gqo_logq_map(float xn, float alpha)
{
    float lam = log1pf(alpha);
    return log1pf(alpha * xn) / lam;
}

float gqo_logq_decode_one(int32_t k, float m, float alpha)
{
    float lam = log1pf(alpha);
    int32_t mag = k < 0 ? -k : k;
    float z = ((float)mag / 127.0f) * lam;
    float x = (expm1f(z) / alpha) * m;
    return k < 0 ? -x : x;
}

int gqo_logq_quantize(const float* x, int W, int nmats, const int64_t* sizes,
                      float alpha, uint64_t seed, uint32_t step,
                      float* maxabs_out, int8_t* codes_out)
{
    return gqo_logq_quantize_workers(x, W, nmats, sizes, alpha, seed, step, 0u,
                                     maxabs_out, codes_out);
}

int gqo_logq_quantize_workers(const float* x, int W, int nmats,
                              const int64_t* sizes, float alpha, uint64_t seed,
                              uint32_t step, uint32_t worker0,
                              float* maxabs_out, int8_t* codes_out)
{
    if (!x || !sizes || !maxabs_out || !codes_out || W < 1 || nmats < 1)
        return -1;
    if (!(alpha > 0.0f) || !isfinite(alpha)) return -1;
    int64_t total = 0;
    for (int m = 0; m < nmats; ++m) {
        if (sizes[m] < 0) return -1;
        total += sizes[m];
    }
    float lam = log1pf(alpha);
    for (int w = 0; w < W; ++w) {
        int64_t base = (int64_t)w * total;
        for (int m = 0; m < nmats; ++m) {
            const float* xm = x + base;
            int8_t* cm = codes_out + base;
            int64_t nm = sizes[m];
            float mx = 0.0f;
            for (int64_t i = 0; i < nm; ++i) {
                float a = fabsf(xm[i]);
                if (a > mx || isnan(a)) mx = a;
                if (isnan(a)) break;
            }
            maxabs_out[(int64_t)w * nmats + m] = mx;
            int usable = (mx > 0.0f) && isfinite(mx);
            uint32_t tag = 0x4C510000u | (uint32_t)m;
            for (int64_t i = 0; i < nm; ++i) {
                if (!usable) {
                    cm[i] = 0;
                    continue;
                }
                float xn = fabsf(xm[i]) / mx;
                float t = log1pf(alpha * xn) / lam;
                float y = t * 127.0f;
                if (!(y <= 127.0f)) y = 127.0f;
                float l = floorf(y);
                float p = y - l;
                uint32_t f = gqo_uniform_bits(seed, tag, step, worker0 + (uint32_t)w,
                                              (uint64_t)i);
                int32_t k = (int32_t)l + round_up(p, f);
                cm[i] = (int8_t)(sign_negative(xm[i]) ? -k : k);
            }
            base += nm;
        }
    }
    return 0;
}

int gqo_logq_decode_sum(const int8_t* codes, const float* maxabs, int W,
                        int nmats, const int64_t* sizes, float alpha,
                        float* out)
{
    if (!codes || !maxabs || !sizes || !out || W < 1 || nmats < 1) return -1;
    int64_t total = 0;
    for (int m = 0; m < nmats; ++m) total += sizes[m];
    int64_t off = 0;
    for (int m = 0; m < nmats; ++m) {
        for (int64_t i = 0; i < sizes[m]; ++i) {
            float acc = 0.0f;
            for (int w = 0; w < W; ++w) {
                float mx = maxabs[(int64_t)w * nmats + m];
                int32_t k = codes[(int64_t)w * total + off + i];
                acc = acc + gqo_logq_decode_one(k, mx, alpha);
            }
            out[off + i] = acc;
        }
        off += sizes[m];
    }
    return 0;
}

/* PowerSGD's decompression Ghat = P Q^T ("Trustworthy Efficient Communication
 * for Distributed Learning using LQ-SGD Algorithm", review, "What carries the
 * argument": G ~ P Q^T), evaluated in the float32 order the library states. */
void gqo_lowrank_fma(const float* P, const float* Q, int64_t n, int64_t m, int r,
                     float* out)
{
    for (int64_t i = 0; i < n; ++i)
        for (int64_t j = 0; j < m; ++j) {
            float acc = 0.0f;
            for (int k = 0; k < r; ++k) acc = fmaf(P[i * r + k], Q[j * r + k], acc);
            out[i * m + j] = acc;
        }
}

/* ------------------------------------------------------------------------
 * [NC] Natural compression (Horvath, Ho, Horvath, Sahu, Canini, Richtarik,
 * "Natural Compression for Distributed Deep Learning", MSML 2022, cited in
 * the Global-QSGD record): stochastic rounding of |x| to one of the two
 * powers of two around it, p = (|x| - 2^e) / 2^e of going up, so the result
 * is unbiased and its variance (2^(e+1) - |x|)(|x| - 2^e) is at most x^2/8.
 * Values below the smallest normal float have no exponent of their own: they
 * round between 0 and 2^-126, with p = |x| / 2^-126.  The result keeps the
 * sign of x, a zero result included.
 * ---------------------------------------------------------------------- */
static float nat_round(float x, uint32_t f)
{
    float ax = fabsf(x);
    float lower, upper, p;
    if (ax < 0x1p-126f) {
        lower = 0.0f;
        upper = 0x1p-126f;
        p = ldexpf(ax, 126); /* exact: a subnormal has at most 23 significant bits */
    } else {
        int e2;
        (void)frexpf(ax, &e2); /* ax = m * 2^e2 with m in [0.5, 1) */
        lower = ldexpf(1.0f, e2 - 1);
        upper = ldexpf(1.0f, e2); /* 2^128 overflows to infinity */
        p = ax / lower - 1.0f;    /* exact: in [0, 1) with at most 23 fraction bits */
    }
    float mag = round_up(p, f) ? upper : lower;
    return sign_negative(x) ? -mag : mag;
}

/* Sign and biased exponent of a signed power of two, zero or infinity: by
 * definition the top nine bits of its IEEE-754 binary32 pattern. */
static uint16_t nat_code_of(float v)
{
    uint32_t bits;
    memcpy(&bits, &v, sizeof bits);
    return (uint16_t)(bits >> 23);
}

int gqo_nat_quantize_workers(const float* x, int W, int64_t n, const int64_t* js,
                             uint32_t worker0, uint64_t seed, uint32_t step,
                             uint16_t* codes_out)
{
    if (!x || !codes_out || W < 1 || n < 0) return -1;
    for (int w = 0; w < W; ++w) {
        for (int64_t i = 0; i < n; ++i) {
            int64_t at = (int64_t)w * n + i;
            uint64_t j = js ? (uint64_t)js[i] : (uint64_t)i;
            uint32_t f = gqo_uniform_bits(seed, GQO_NAT_TAG, step, worker0 + (uint32_t)w, j);
            codes_out[at] = nat_code_of(nat_round(x[at], f));
        }
    }
    return 0;
}

float gqo_nat_value(uint16_t code)
{
    int E = code & 0xFF;
    float mag = E == 0 ? 0.0f : (E == 255 ? INFINITY : ldexpf(1.0f, E - 127));
    return (code & 0x100) ? -mag : mag;
}

int gqo_nat_decode(const uint16_t* codes, int64_t n, float* out)
{
    if (!codes || !out || n < 0) return -1;
    for (int64_t i = 0; i < n; ++i) out[i] = gqo_nat_value(codes[i]);
    return 0;
}

int gqo_nat_decode_sum(const uint16_t* codes, int W, int64_t n, float* out)
{
    if (!codes || !out || W < 1 || n < 0) return -1;
    for (int64_t i = 0; i < n; ++i) {
        float acc = gqo_nat_value(codes[i]);
        for (int w = 1; w < W; ++w) acc = acc + gqo_nat_value(codes[(int64_t)w * n + i]);
        out[i] = acc;
    }
    return 0;
}

