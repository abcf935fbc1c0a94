// gq_api.cu -- host side of the libgq C ABI: argument checks, launch shapes,
// and the composition of the kernels into the calls declared in gq_api.h.
#include <cuda_runtime.h>

#include <cstdint>
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "gq_api.h"
#include "gq_internal.h"
#include "gq_psgd.h"
#include "gq_nat.h"

namespace gq {
// The log map's division as the quantize kernel computes it (gq_logq.cu).
cudaError_t launch_fma_div_selftest(const float* a, float b, float* out, long long n, int sms,
                                    cudaStream_t st);
}  // namespace gq

using namespace gq;

namespace {

// An NVTX range around each compute call of the ABI (free when no tool is
// attached), so that timelines and profiles show the library's calls.
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};

constexpr int kVersion = 100;  // 0.1.0

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned8(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 7u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// Streaming multiprocessors of the current device (cached per device).
int sm_count() {
    static std::mutex mu;
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    std::lock_guard<std::mutex> lock(mu);
    if (cached[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

// Resident 256-thread blocks per SM the streaming kernels are sized for.
constexpr int kBlocksPerSm = 8;

int max_code(const gq_config& c) { return c.levels == GQ_UNIFORM ? c.s : c.L; }

// Largest value one worker adds to the sum (in the sum's units).
long long max_value(const gq_config& c) {
    return c.levels == GQ_UNIFORM ? (long long)c.s : (1LL << (c.L - 1));
}

int check_levels(const gq_config* c) {
    if (!c) return GQ_ERR_ARG;
    if (c->levels == GQ_UNIFORM) {
        if (c->s < 1 || c->s > 32767) return GQ_ERR_ARG;
    } else if (c->levels == GQ_EXP) {
        if (c->L < 1 || c->L > 15) return GQ_ERR_ARG;
    } else {
        return GQ_ERR_ARG;
    }
    return GQ_OK;
}

int check_bits(const gq_config* c) {
    if (c->bits != 4 && c->bits != 5 && c->bits != 8 && c->bits != 16) return GQ_ERR_ARG;
    // codes -max..max need 2*max+1 distinct two's-complement values
    const long long need = 2LL * max_code(*c) + 1;
    if (need > (1LL << c->bits)) return GQ_ERR_ARG;
    return GQ_OK;
}

int check_wire(const gq_config* c, int W) {
    if (c->wire != GQ_WIRE_INT8 && c->wire != GQ_WIRE_INT16 && c->wire != GQ_WIRE_F16)
        return GQ_ERR_ARG;
    const long long lim = c->wire == GQ_WIRE_INT8 ? 127 : c->wire == GQ_WIRE_INT16 ? 32767 : 2048;
    if ((long long)W * max_value(*c) > lim) return GQ_ERR_OVERFLOW;
    return GQ_OK;
}

int check_scale_kind(const gq_config* c) {
    return (c->scale_kind == GQ_SCALE_L2 || c->scale_kind == GQ_SCALE_MAXABS) ? GQ_OK : GQ_ERR_ARG;
}

int check_sizes(int W, long long d) {
    if (W < 1 || d < 0) return GQ_ERR_ARG;
    // codes rows, offsets and Philox counters are 64-bit; keep W*d addressable
    if (d > (1LL << 40) || (long long)W * d > (1LL << 42)) return GQ_ERR_ARG;
    return GQ_OK;
}

int stream_grid(long long d);

// The bulk-copy pipeline of the fused pass: stages per block (compile-time
// knob), and whether it is used at all.
#ifndef GQ_TMA_STAGES
#define GQ_TMA_STAGES 3
#endif
#ifndef GQ_USE_TMA
#define GQ_USE_TMA 1
#endif
constexpr size_t kSmemPerBlockMax = 232448;  // 227 KiB of dynamic shared memory
constexpr size_t kSmemPerSm = 233472;        // 228 KiB per SM, 1 KiB reserved per block

// Stages that fit one block for W rows (2W with error feedback), or 0 when the
// rows do not fit even two stages (then the register-staged kernel runs).
int tma_stages(int W, bool ef) {
    for (int s = GQ_TMA_STAGES; s >= 2; --s)
        if (tma_smem_bytes(W, ef, s) <= kSmemPerBlockMax) return s;
    return 0;
}

int tma_grid(long long d, int W, bool ef, int stages) {
    const long long tiles = (d + 1023) / 1024;
    long long per_sm = (long long)(kSmemPerSm / (tma_smem_bytes(W, ef, stages) + 1024));
    if (per_sm < 1) per_sm = 1;
    const long long cap = (long long)sm_count() * per_sm;
    const long long g = tiles < cap ? tiles : cap;
    return g < 1 ? 1 : (int)g;
}

// Launch the fused pass on the best path for the shape.
cudaError_t launch_fused(QuantArgs& a, int levels, int bits, bool ef_read, void* ws, long long d,
                         cudaStream_t stream) {
    const bool vec = (d % 4) == 0;
    const int stages = (GQ_USE_TMA && vec) ? tma_stages(a.W, ef_read) : 0;
    a.hdr = reinterpret_cast<WsHeader*>(ws);
    if (stages > 0)
        return launch_quant_tma(a, levels, bits, ef_read, stages,
                                tma_grid(d, a.W, ef_read, stages), stream);
    return launch_quant(a, levels, bits, ef_read, vec, stream_grid(d), stream);
}

int stream_grid(long long d) {
    const long long blocks128 = (d + 127) / 128;                 // one warp each
    const long long need = (blocks128 + (kThreads / 32) - 1) / (kThreads / 32);
    const long long cap = (long long)sm_count() * kBlocksPerSm;
    long long g = need < cap ? need : cap;
    return g < 1 ? 1 : (int)g;
}

void round_keys(unsigned long long seed, uint32_t tag, RoundKeys& rk) {
    uint32_t k0 = (uint32_t)seed, k1 = (uint32_t)(seed >> 32) ^ tag;
    for (int r = 0; r < 10; ++r) {
        rk.k[2 * r] = k0;
        rk.k[2 * r + 1] = k1;
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
}

long long row_bytes_of(int bits, long long d) { return ((d + 127) / 128) * 16LL * bits; }

bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

int cuda_status(cudaError_t e) { return e == cudaSuccess ? GQ_OK : GQ_ERR_CUDA; }

WsHeader* header_of(void* ws) { return reinterpret_cast<WsHeader*>(ws); }
unsigned long long* partials_of(void* ws) {
    return reinterpret_cast<unsigned long long*>(reinterpret_cast<char*>(ws) + kWorkspaceHeader);
}

void fill_quant_args(QuantArgs& a, const gq_config* cfg, int W, long long d) {
    std::memset(&a, 0, sizeof(a));
    round_keys(cfg->seed, 0u, a.rk);
    a.d = d;
    a.W = W;
    a.wire = cfg->wire;
    a.step = cfg->step;
    a.worker0 = cfg->worker0;
    a.q0 = cfg->coord0 >> 2;
    a.step_dev = cfg->step_dev;
    a.L = cfg->L;
    a.smax = (float)cfg->s;
    a.finest = cfg->levels == GQ_EXP ? std::ldexp(1.0f, -(cfg->L - 1)) : 1.0f;
    a.inv_finest = cfg->levels == GQ_EXP ? std::ldexp(1.0f, cfg->L - 1) : 1.0f;
    a.exp_shift = cfg->levels == GQ_EXP ? std::ldexp(1.0f, cfg->L - 127) : 1.0f;
    a.w_pow2 = is_pow2(W) ? 1 : 0;
    a.inv_w = a.w_pow2 ? 1.0f / (float)W : 0.0f;
}

// Per-bucket scales: buckets of 2^b coordinates, partials per chunk of
// 2^min(b, 12) coordinates.
constexpr int kBucketLog2Min = 7, kBucketLog2Max = 30, kChunkLog2Max = 12;

int chunk_log2_of(int b) { return b < kChunkLog2Max ? b : kChunkLog2Max; }
long long count_of(long long d, int log2) { return (d + (1LL << log2) - 1) >> log2; }

size_t bucket_ws_bytes(int W, long long d, int b) {
    const size_t items = (size_t)W * (size_t)count_of(d, chunk_log2_of(b));
    const size_t own = kWorkspaceHeader + items * (sizeof(double) + sizeof(unsigned));
    const size_t global = kWorkspaceHeader + (size_t)W * kMaxNormBlocks * 2 * sizeof(double);
    const size_t n = own > global ? own : global;
    return (n + 255) & ~(size_t)255;
}

}  // namespace

namespace gq {

// Blocks per worker of the norm pass: one full wave of resident blocks over
// all workers, so that no block starts late and leaves a tail.  The fp32 runs
// and the fp64 combine order follow from this count, so every caller of the
// norm kernel that wants gq_global_norm's exact scale uses it.
int norm_blocks_per_worker(int W, long long d, int kind, bool has_e) {
    const long long resident = (long long)sm_count() * norm_resident_blocks(kind, has_e, d % 4 == 0);
    const long long want = resident / W > 0 ? resident / W : 1;
    const long long useful = (d + (long long)kThreads * 16 - 1) / ((long long)kThreads * 16);
    long long nb = want < useful ? want : useful;
    if (nb < 1) nb = 1;
    if (nb > kMaxNormBlocks) nb = kMaxNormBlocks;
    return (int)nb;
}

}  // namespace gq

extern "C" {

GQ_API int gq_version(void) { return kVersion; }

GQ_API const char* gq_status_string(int status) {
    switch (status) {
        case GQ_OK: return "ok";
        case GQ_ERR_ARG: return "invalid argument";
        case GQ_ERR_OVERFLOW: return "W * max code value overflows the sum type";
        case GQ_ERR_ALIGN: return "buffer not 16-byte aligned";
        case GQ_ERR_CUDA: return "CUDA error";
        case GQ_ERR_NONFINITE: return "non-finite scale (NaN or Inf in the input)";
        case GQ_ERR_SIZE: return "size beyond the fixed maximum of this entry point";
        case GQ_ERR_TIMEOUT: return "a bounded wait inside a kernel expired";
        default: return "unknown status";
    }
}

GQ_API int gq_advance_step(unsigned int* step_dev, unsigned int by, cudaStream_t stream) {
    if (!step_dev) return GQ_ERR_ARG;
    if (!aligned4(step_dev)) return GQ_ERR_ALIGN;
    return cuda_status(launch_advance_step(step_dev, by, stream));
}

GQ_API int gq_validate(const gq_config* cfg, int W, long long d) {
    if (!cfg || (cfg->coord0 & 3ull) != 0) return GQ_ERR_ARG;
    if (cfg->step_dev && !aligned4(cfg->step_dev)) return GQ_ERR_ALIGN;
    int rc = check_levels(cfg);
    if (rc) return rc;
    if ((rc = check_sizes(W, d))) return rc;
    if ((rc = check_bits(cfg))) return rc;
    if ((rc = check_scale_kind(cfg))) return rc;
    if (cfg->ef != 0 && cfg->ef != 1) return GQ_ERR_ARG;
    return check_wire(cfg, W);
}

GQ_API int gq_packed_row_bytes(const gq_config* cfg, long long d, long long* bytes) {
    if (!cfg || !bytes || d < 0) return GQ_ERR_ARG;
    if (cfg->bits != 4 && cfg->bits != 5 && cfg->bits != 8 && cfg->bits != 16) return GQ_ERR_ARG;
    *bytes = row_bytes_of(cfg->bits, d);
    return GQ_OK;
}

GQ_API int gq_workspace_bytes(const gq_config* cfg, int W, long long d, size_t* bytes) {
    (void)cfg;
    if (!bytes || W < 1 || d < 0) return GQ_ERR_ARG;
    *bytes = (size_t)kWorkspaceHeader + (size_t)W * kMaxNormBlocks * 2 * sizeof(unsigned long long);
    return GQ_OK;
}

GQ_API int gq_workspace_init(void* ws_dev, size_t bytes, cudaStream_t stream) {
    if (!ws_dev || bytes < (size_t)kWorkspaceHeader) return GQ_ERR_ARG;
    if (!aligned16(ws_dev)) return GQ_ERR_ALIGN;
    return cuda_status(cudaMemsetAsync(ws_dev, 0, bytes, stream));
}

GQ_API int gq_get_device_status(void* ws_dev, cudaStream_t stream) {
    if (!ws_dev) return GQ_ERR_ARG;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return GQ_ERR_CUDA;
    unsigned int flags = 0;
    if (cudaMemcpy(&flags, &header_of(ws_dev)->flags, sizeof(flags), cudaMemcpyDeviceToHost) !=
        cudaSuccess)
        return GQ_ERR_CUDA;
    if (flags == 0) return GQ_OK;
    if (cudaMemset(&header_of(ws_dev)->flags, 0, sizeof(flags)) != cudaSuccess) return GQ_ERR_CUDA;
    return (flags & kFlagPipelineTimeout) ? GQ_ERR_TIMEOUT : GQ_ERR_NONFINITE;
}

GQ_API int gq_selftest_wait_timeout(void* ws_dev, unsigned int limit_ms, cudaStream_t stream) {
    if (!ws_dev || limit_ms < 1 || limit_ms > 10000) return GQ_ERR_ARG;
    if (!aligned16(ws_dev)) return GQ_ERR_ALIGN;
    return cuda_status(launch_wait_timeout_selftest(header_of(ws_dev),
                                                    (unsigned long long)limit_ms * 1000000ull,
                                                    stream));
}

GQ_API int gq_selftest_fma_div(const float* a_dev, float b, float* out_dev, long long n,
                               cudaStream_t stream) {
    if (n < 0 || (n > 0 && (!a_dev || !out_dev)) || !(b > 0.f) || !(b <= 3.4028235e38f))
        return GQ_ERR_ARG;
    if (!aligned4(a_dev) || !aligned4(out_dev)) return GQ_ERR_ALIGN;
    if (n == 0) return GQ_OK;
    return cuda_status(launch_fma_div_selftest(a_dev, b, out_dev, n, sm_count(), stream));
}

GQ_API int gq_global_norm(const float* g_dev, const float* e_dev, int W, long long d,
                          const gq_config* cfg, float* scale_dev, double* norms_dev, void* ws_dev,
                          cudaStream_t stream) {
    const NvtxRange nvtx_range("gq_global_norm");
    if (!cfg || (!g_dev && d > 0) || !scale_dev || !ws_dev) return GQ_ERR_ARG;
    int rc = check_sizes(W, d);
    if (rc) return rc;
    if ((rc = check_scale_kind(cfg))) return rc;
    if (cfg->ef && !e_dev && d > 0) return GQ_ERR_ARG;
    if (!aligned16(g_dev) || (e_dev && !aligned16(e_dev)) || !aligned16(ws_dev) ||
        !aligned4(scale_dev) || (norms_dev && !aligned8(norms_dev)))
        return GQ_ERR_ALIGN;
    NormArgs a;
    a.g = g_dev;
    a.e = cfg->ef ? e_dev : nullptr;
    a.d = d;
    a.W = W;
    a.nb = norm_blocks_per_worker(W, d, cfg->scale_kind, cfg->ef != 0);
    a.kind = cfg->scale_kind;
    a.scale = scale_dev;
    a.norms = norms_dev;
    a.partials = partials_of(ws_dev);
    a.hdr = header_of(ws_dev);
    return cuda_status(launch_norm(a, (d % 4) == 0, stream));
}

static int quant_common(const float* g_dev, float* e_dev, int W, long long d, const gq_config* cfg,
                        const float* scale_dev, void* codes_dev, void* sum_dev, float* out_dev,
                        void* ws_dev, bool allow_ef, cudaStream_t stream) {
    int rc = gq_validate(cfg, W, d);
    if (rc) return rc;
    if (!g_dev || !scale_dev || !ws_dev) return GQ_ERR_ARG;
    const bool ef = allow_ef && cfg->ef;
    if (ef && !e_dev) return GQ_ERR_ARG;
    if (!codes_dev && !sum_dev && !out_dev && !ef) return GQ_ERR_ARG;
    if (!aligned16(g_dev) || (ef && !aligned16(e_dev)) || !aligned4(scale_dev) ||
        (codes_dev && !aligned16(codes_dev)) || (sum_dev && !aligned16(sum_dev)) ||
        (out_dev && !aligned16(out_dev)))
        return GQ_ERR_ALIGN;
    if (d == 0) return GQ_OK;
    QuantArgs a;
    fill_quant_args(a, cfg, W, d);
    a.g = g_dev;
    a.e = ef ? e_dev : nullptr;
    a.scale = scale_dev;
    a.codes = reinterpret_cast<unsigned char*>(codes_dev);
    a.row_bytes = row_bytes_of(cfg->bits, d);
    a.update_e = ef ? 1 : 0;
    a.sum = sum_dev;
    a.out = out_dev;
    const int bits = codes_dev ? cfg->bits : 0;
    return cuda_status(launch_fused(a, cfg->levels, bits, ef, ws_dev, d, stream));
}

GQ_API int gq_quantize_pack(const float* g_dev, const float* e_dev, int W, long long d,
                            const gq_config* cfg, const float* scale_dev, void* codes_dev,
                            void* ws_dev, cudaStream_t stream) {
    const NvtxRange nvtx_range("gq_quantize_pack");
    if (!codes_dev) return GQ_ERR_ARG;
    // v = g + e is read but e is not updated here: the update belongs to step 5
    gq_config c;
    if (!cfg) return GQ_ERR_ARG;
    c = *cfg;
    if (c.ef && !e_dev) return GQ_ERR_ARG;
    if (c.ef && !aligned16(e_dev)) return GQ_ERR_ALIGN;
    int rc = gq_validate(&c, W, d);
    if (rc) return rc;
    if (!g_dev || !scale_dev || !ws_dev) return GQ_ERR_ARG;
    if (!aligned16(g_dev) || !aligned4(scale_dev) || !aligned16(codes_dev)) return GQ_ERR_ALIGN;
    if (d == 0) return GQ_OK;
    QuantArgs a;
    fill_quant_args(a, &c, W, d);
    a.g = g_dev;
    a.e = c.ef ? const_cast<float*>(e_dev) : nullptr;  // read only: update_e = 0
    a.update_e = 0;
    a.scale = scale_dev;
    a.codes = reinterpret_cast<unsigned char*>(codes_dev);
    a.row_bytes = row_bytes_of(c.bits, d);
    return cuda_status(launch_fused(a, c.levels, c.bits, c.ef != 0, ws_dev, d, stream));
}

GQ_API int gq_aggregate(const void* codes_dev, int W, long long d, const gq_config* cfg,
                        void* sum_dev, void* ws_dev, cudaStream_t stream) {
    const NvtxRange nvtx_range("gq_aggregate");
    (void)ws_dev;
    int rc = gq_validate(cfg, W, d);
    if (rc) return rc;
    if (!codes_dev || !sum_dev) return GQ_ERR_ARG;
    if (!aligned16(codes_dev) || !aligned16(sum_dev)) return GQ_ERR_ALIGN;
    if (d == 0) return GQ_OK;
    AggArgs a;
    a.codes = reinterpret_cast<const unsigned char*>(codes_dev);
    a.row_bytes = row_bytes_of(cfg->bits, d);
    a.sum = sum_dev;
    a.d = d;
    a.W = W;
    a.wire = cfg->wire;
    return cuda_status(launch_aggregate(a, cfg->levels, cfg->bits, stream_grid(d), stream));
}

GQ_API int gq_dequantize_ef(const void* sum_dev, const void* codes_dev, const float* g_dev,
                            float* e_dev, int W, long long d, const gq_config* cfg,
                            const float* scale_dev, float* out_dev, void* ws_dev,
                            cudaStream_t stream) {
    const NvtxRange nvtx_range("gq_dequantize_ef");
    (void)ws_dev;
    int rc = gq_validate(cfg, W, d);
    if (rc) return rc;
    if (!scale_dev) return GQ_ERR_ARG;
    const bool dec = sum_dev != nullptr;
    const bool ef = cfg->ef && e_dev;
    if (dec && !out_dev) return GQ_ERR_ARG;
    if (!dec && !ef) return GQ_ERR_ARG;
    if (ef && (!codes_dev || !g_dev)) return GQ_ERR_ARG;
    if (!aligned4(scale_dev) || (dec && (!aligned16(sum_dev) || !aligned16(out_dev))) ||
        (ef && (!aligned16(codes_dev) || !aligned16(g_dev) || !aligned16(e_dev))))
        return GQ_ERR_ALIGN;
    if (d == 0) return GQ_OK;
    DequantArgs a;
    a.sum = dec ? sum_dev : nullptr;
    a.codes = reinterpret_cast<const unsigned char*>(codes_dev);
    a.row_bytes = row_bytes_of(cfg->bits, d);
    a.g = g_dev;
    a.e = ef ? e_dev : nullptr;
    a.scale = scale_dev;
    a.out = out_dev;
    a.d = d;
    a.W = W;
    a.wire = cfg->wire;
    a.smax = (float)cfg->s;
    a.finest = cfg->levels == GQ_EXP ? std::ldexp(1.0f, -(cfg->L - 1)) : 1.0f;
    a.w_pow2 = is_pow2(W) ? 1 : 0;
    a.inv_w = a.w_pow2 ? 1.0f / (float)W : 0.0f;
    return cuda_status(
        launch_dequant(a, cfg->levels, cfg->bits, (d % 4) == 0, stream_grid(d), stream));
}

GQ_API int gq_quantize_aggregate(const float* g_dev, float* e_dev, int W, long long d,
                                 const gq_config* cfg, const float* scale_dev, void* codes_dev,
                                 void* sum_dev, float* out_dev, void* ws_dev, cudaStream_t stream) {
    const NvtxRange nvtx_range("gq_quantize_aggregate");
    return quant_common(g_dev, e_dev, W, d, cfg, scale_dev, codes_dev, sum_dev, out_dev, ws_dev,
                        true, stream);
}

GQ_API int gq_step_fused(const float* g_dev, float* e_dev, int W, long long d,
                         const gq_config* cfg, float* scale_dev, double* norms_dev,
                         void* codes_dev, void* sum_dev, float* out_dev, void* ws_dev,
                         cudaStream_t stream) {
    const NvtxRange nvtx_range("gq_step_fused");
    int rc = gq_validate(cfg, W, d);
    if (rc) return rc;
    if (cfg->ef && !e_dev) return GQ_ERR_ARG;
    if (!codes_dev && !sum_dev && !out_dev && !cfg->ef) return GQ_ERR_ARG;
    if (!aligned16(g_dev) || (cfg->ef && !aligned16(e_dev)) ||
        (codes_dev && !aligned16(codes_dev)) || (sum_dev && !aligned16(sum_dev)) ||
        (out_dev && !aligned16(out_dev)))
        return GQ_ERR_ALIGN;
    rc = gq_global_norm(g_dev, cfg->ef ? e_dev : nullptr, W, d, cfg, scale_dev, norms_dev, ws_dev,
                        stream);
    if (rc) return rc;
    return gq_quantize_aggregate(g_dev, e_dev, W, d, cfg, scale_dev, codes_dev, sum_dev, out_dev,
                                 ws_dev, stream);
}

GQ_API int gq_step_fused_host(const float* g_host, float* g_dev, float* e_dev, int W, long long d,
                              const gq_config* cfg, float* scale_dev, void* codes_dev,
                              void* sum_dev, float* out_dev, float* out_host, float* scale_host,
                              void* ws_dev, cudaStream_t stream) {
    const NvtxRange nvtx_range("gq_step_fused_host");
    int rc = gq_validate(cfg, W, d);
    if (rc) return rc;
    if (!g_host || !g_dev || !out_dev || !out_host) return GQ_ERR_ARG;
    const size_t gbytes = (size_t)W * (size_t)d * sizeof(float);
    if (cudaMemcpyAsync(g_dev, g_host, gbytes, cudaMemcpyHostToDevice, stream) != cudaSuccess)
        return GQ_ERR_CUDA;
    rc = gq_step_fused(g_dev, e_dev, W, d, cfg, scale_dev, nullptr, codes_dev, sum_dev, out_dev,
                       ws_dev, stream);
    if (rc) return rc;
    if (cudaMemcpyAsync(out_host, out_dev, (size_t)d * sizeof(float), cudaMemcpyDeviceToHost,
                        stream) != cudaSuccess)
        return GQ_ERR_CUDA;
    if (scale_host && cudaMemcpyAsync(scale_host, scale_dev, sizeof(float), cudaMemcpyDeviceToHost,
                                      stream) != cudaSuccess)
        return GQ_ERR_CUDA;
    return GQ_OK;
}

static int logq_offsets(int nmats, const int* rows, const int* cols, long long* total) {
    if (nmats < 1 || nmats > 4096 || !rows || !cols) return GQ_ERR_ARG;
    long long t = 0;
    for (int m = 0; m < nmats; ++m) {
        if (rows[m] < 0 || cols[m] < 0) return GQ_ERR_ARG;
        t += (long long)rows[m] * cols[m];
    }
    *total = t;
    return GQ_OK;
}

static void logq_group(LogqArgs& a, int m0, int count, const int* rows, const int* cols) {
    a.m0 = m0;
    a.count = count;
    long long off = 0;
    for (int m = 0; m < m0; ++m) off += (long long)rows[m] * cols[m];
    a.off[0] = off;
    for (int i = 0; i < count; ++i) a.off[i + 1] = a.off[i] + (long long)rows[m0 + i] * cols[m0 + i];
}

GQ_API int gq_nat_quantize(const float* x_dev, int W, long long n, const gq_config* cfg,
                           unsigned short* codes_dev, void* ws_dev, cudaStream_t stream) {
    const NvtxRange nvtx_range("gq_nat_quantize");
    if (!cfg || cfg->levels != GQ_NAT || !ws_dev || W > 65535) return GQ_ERR_ARG;
    int rc = check_sizes(W, n);
    if (rc) return rc;
    if (n > 0 && (!x_dev || !codes_dev)) return GQ_ERR_ARG;
    if (!aligned16(x_dev) || !aligned16(codes_dev) || !aligned16(ws_dev) ||
        (cfg->step_dev && !aligned4(cfg->step_dev)))
        return GQ_ERR_ALIGN;
    if (n == 0) return GQ_OK;
    NatArgs a;
    std::memset(&a, 0, sizeof(a));
    a.x = x_dev;
    a.codes = codes_dev;
    a.n = n;
    a.W = W;
    a.worker0 = cfg->worker0;
    a.step = cfg->step;
    a.step_dev = cfg->step_dev;
    round_keys(cfg->seed, kNatTag, a.rk);
    a.hdr = header_of(ws_dev);
    return cuda_status(launch_nat_quantize(a, (n % 4) == 0, sm_count(), stream));
}

GQ_API int gq_nat_decode_sum(const unsigned short* codes_dev, int W, long long n,
                             float* out_dev, cudaStream_t stream) {
    const NvtxRange nvtx_range("gq_nat_decode_sum");
    int rc = check_sizes(W, n);
    if (rc) return rc;
    if (n > 0 && (!codes_dev || !out_dev)) return GQ_ERR_ARG;
    if (!aligned16(codes_dev) || !aligned16(out_dev)) return GQ_ERR_ALIGN;
    if (n == 0) return GQ_OK;
    NatArgs a;
    std::memset(&a, 0, sizeof(a));
    a.ccodes = codes_dev;
    a.out = out_dev;
    a.n = n;
    a.W = W;
    return cuda_status(launch_nat_decode_sum(a, (n % 4) == 0, sm_count(), stream));
}

GQ_API int gq_logq_quantize(const float* x_dev, int W, int nmats, const int* rows_host,
                            const int* cols_host, const gq_config* cfg, float* maxabs_dev,
                            signed char* codes_dev, void* ws_dev, cudaStream_t stream) {
    const NvtxRange nvtx_range("gq_logq_quantize");
    if (!cfg || cfg->levels != GQ_LOG || !(cfg->alpha > 0.f) || !(cfg->alpha <= 3.0e38f))
        return GQ_ERR_ARG;
    if (!x_dev || !maxabs_dev || !codes_dev || !ws_dev || W < 1) return GQ_ERR_ARG;
    long long total = 0;
    int rc = logq_offsets(nmats, rows_host, cols_host, &total);
    if (rc) return rc;
    if (!aligned16(x_dev) || !aligned4(maxabs_dev) || !aligned16(ws_dev)) return GQ_ERR_ALIGN;
    LogqArgs a;
    std::memset(&a, 0, sizeof(a));
    a.x = x_dev;
    a.codes = codes_dev;
    a.maxabs = maxabs_dev;
    a.total = total;
    a.W = W;
    a.nmats = nmats;
    a.step = cfg->step;
    a.worker0 = cfg->worker0;
    a.step_dev = cfg->step_dev;
    a.seed_lo = (uint32_t)cfg->seed;
    a.seed_hi = (uint32_t)(cfg->seed >> 32);
    a.alpha = cfg->alpha;
    a.hdr = header_of(ws_dev);
    for (int m0 = 0; m0 < nmats; m0 += kLogqGroup) {
        const int count = nmats - m0 < kLogqGroup ? nmats - m0 : kLogqGroup;
        logq_group(a, m0, count, rows_host, cols_host);
        if ((rc = cuda_status(launch_logq_quantize(a, stream)))) return rc;
    }
    return GQ_OK;
}

GQ_API int gq_logq_decode_sum(const signed char* codes_dev, const float* maxabs_dev, int W,
                              int nmats, const int* rows_host, const int* cols_host,
                              const gq_config* cfg, float* out_dev, cudaStream_t stream) {
    const NvtxRange nvtx_range("gq_logq_decode_sum");
    if (!cfg || cfg->levels != GQ_LOG || !(cfg->alpha > 0.f) || !(cfg->alpha <= 3.0e38f))
        return GQ_ERR_ARG;
    if (!codes_dev || !maxabs_dev || !out_dev || W < 1) return GQ_ERR_ARG;
    long long total = 0;
    int rc = logq_offsets(nmats, rows_host, cols_host, &total);
    if (rc) return rc;
    if (!aligned4(maxabs_dev) || !aligned4(out_dev)) return GQ_ERR_ALIGN;
    LogqArgs a;
    std::memset(&a, 0, sizeof(a));
    a.ccodes = codes_dev;
    a.cmaxabs = maxabs_dev;
    a.out = out_dev;
    a.total = total;
    a.W = W;
    a.nmats = nmats;
    a.alpha = cfg->alpha;
    for (int m0 = 0; m0 < nmats; m0 += kLogqGroup) {
        const int count = nmats - m0 < kLogqGroup ? nmats - m0 : kLogqGroup;
        logq_group(a, m0, count, rows_host, cols_host);
        if ((rc = cuda_status(launch_logq_decode(a, stream)))) return rc;
    }
    return GQ_OK;
}

GQ_API int gq_bucket_count(long long d, int bucket_log2, long long* nbuckets) {
    if (!nbuckets || d < 0 || bucket_log2 < kBucketLog2Min || bucket_log2 > kBucketLog2Max)
        return GQ_ERR_ARG;
    *nbuckets = count_of(d, bucket_log2);
    return GQ_OK;
}

GQ_API int gq_bucket_workspace_bytes(const gq_config* cfg, int W, long long d, int bucket_log2,
                                     size_t* bytes) {
    if (!cfg || !bytes || bucket_log2 < kBucketLog2Min || bucket_log2 > kBucketLog2Max)
        return GQ_ERR_ARG;
    int rc = check_sizes(W, d);
    if (rc) return rc;
    *bytes = bucket_ws_bytes(W, d, bucket_log2);
    return GQ_OK;
}

GQ_API int gq_bucket_scales(const float* g_dev, const float* e_dev, int W, long long d,
                            int bucket_log2, const gq_config* cfg, float* table_dev, void* ws_dev,
                            cudaStream_t stream) {
    const NvtxRange nvtx_range("gq_bucket_scales");
    if (!cfg || bucket_log2 < kBucketLog2Min || bucket_log2 > kBucketLog2Max) return GQ_ERR_ARG;
    int rc = gq_validate(cfg, W, d);
    if (rc) return rc;
    if (cfg->levels == GQ_LOG) return GQ_ERR_ARG;
    if ((!g_dev && d > 0) || !ws_dev || (!table_dev && d > 0)) return GQ_ERR_ARG;
    if (cfg->ef && !e_dev && d > 0) return GQ_ERR_ARG;
    if (!aligned16(g_dev) || (cfg->ef && !aligned16(e_dev)) || !aligned16(ws_dev) ||
        !aligned4(table_dev))
        return GQ_ERR_ALIGN;
    if (d == 0) return GQ_OK;
    BucketArgs a;
    std::memset(&a, 0, sizeof(a));
    a.g = g_dev;
    a.e = cfg->ef ? e_dev : nullptr;
    a.d = d;
    a.W = W;
    a.bucket_log2 = bucket_log2;
    a.chunk_log2 = chunk_log2_of(bucket_log2);
    a.nbuckets = count_of(d, bucket_log2);
    a.nchunks = count_of(d, a.chunk_log2);
    a.kind = cfg->scale_kind;
    a.levels = cfg->levels;
    a.smax = (float)cfg->s;
    a.finest = cfg->levels == GQ_EXP ? std::ldexp(1.0f, -(cfg->L - 1)) : 1.0f;
    a.scales = table_dev;
    a.mult = table_dev + a.nbuckets;
    a.unit = table_dev + 2 * a.nbuckets;
    a.part_sum = reinterpret_cast<double*>(partials_of(ws_dev));
    a.part_max = reinterpret_cast<unsigned*>(a.part_sum + (size_t)W * a.nchunks);
    a.hdr = header_of(ws_dev);
    return cuda_status(launch_bucket_scales(a, sm_count(), stream));
}

GQ_API int gq_quantize_aggregate_bucketed(const float* g_dev, float* e_dev, int W, long long d,
                                          int bucket_log2, const gq_config* cfg,
                                          const float* table_dev, void* codes_dev, void* sum_dev,
                                          float* out_dev, void* ws_dev, cudaStream_t stream) {
    const NvtxRange nvtx_range("gq_quantize_aggregate_bucketed");
    if (!cfg || bucket_log2 < kBucketLog2Min || bucket_log2 > kBucketLog2Max) return GQ_ERR_ARG;
    int rc = gq_validate(cfg, W, d);
    if (rc) return rc;
    if (cfg->levels == GQ_LOG) return GQ_ERR_ARG;
    if (!g_dev || !table_dev || !ws_dev) return GQ_ERR_ARG;
    const bool ef = cfg->ef != 0;
    if (ef && !e_dev) return GQ_ERR_ARG;
    if (!codes_dev && !sum_dev && !out_dev && !ef) return GQ_ERR_ARG;
    if (!aligned16(g_dev) || (ef && !aligned16(e_dev)) || !aligned4(table_dev) ||
        (codes_dev && !aligned16(codes_dev)) || (sum_dev && !aligned16(sum_dev)) ||
        (out_dev && !aligned16(out_dev)))
        return GQ_ERR_ALIGN;
    if (d == 0) return GQ_OK;
    const long long K = count_of(d, bucket_log2);
    QuantArgs a;
    fill_quant_args(a, cfg, W, d);
    a.g = g_dev;
    a.e = ef ? e_dev : nullptr;
    a.scale = table_dev;  // replaced per 128-coordinate block by the bucket's entries
    a.bq_mult = table_dev + K;
    a.bq_unit = table_dev + 2 * K;
    a.bucket_shift = bucket_log2 - 7;
    a.codes = reinterpret_cast<unsigned char*>(codes_dev);
    a.row_bytes = row_bytes_of(cfg->bits, d);
    a.update_e = ef ? 1 : 0;
    a.sum = sum_dev;
    a.out = out_dev;
    const int bits = codes_dev ? cfg->bits : 0;
    return cuda_status(launch_fused(a, cfg->levels, bits, ef, ws_dev, d, stream));
}

GQ_API int gq_step_bucketed(const float* g_dev, float* e_dev, int W, long long d, int bucket_log2,
                            const gq_config* cfg, float* table_dev, void* codes_dev, void* sum_dev,
                            float* out_dev, void* ws_dev, cudaStream_t stream) {
    const NvtxRange nvtx_range("gq_step_bucketed");
    int rc = gq_bucket_scales(g_dev, cfg && cfg->ef ? e_dev : nullptr, W, d, bucket_log2, cfg,
                              table_dev, ws_dev, stream);
    if (rc) return rc;
    return gq_quantize_aggregate_bucketed(g_dev, e_dev, W, d, bucket_log2, cfg, table_dev,
                                          codes_dev, sum_dev, out_dev, ws_dev, stream);
}

// ---------------------------------------------------------------------------
// PowerSGD low-rank step (LQ-SGD)
// ---------------------------------------------------------------------------
namespace {

// The back projection splits each matrix's rows into chunks so that the whole
// launch has at least this many tiles (about 8 waves of 4 resident blocks on
// 148 SMs, so the last wave's tail stays small); a constant, not the SM count,
// so that the summation order, and hence Q, is the same on every device.
constexpr long long kBackTargetTiles = 4736;

struct PsgdShape {
    int nmats = 0, rank = 0, W = 0, max_rows = 0, chunk_rows = 0, chunks_max = 0;
    const int* rows = nullptr;
    const int* cols = nullptr;
    long long total = 0, ptotal = 0, qtotal = 0;
    bool vec = true;
};

int psgd_shape(int W, int nmats, const int* rows, const int* cols, int rank, PsgdShape& s) {
    if (W < 1 || nmats < 1 || nmats > 4096 || !rows || !cols || rank < 1 || rank > 8)
        return GQ_ERR_ARG;
    s.W = W;
    s.nmats = nmats;
    s.rows = rows;
    s.cols = cols;
    s.rank = rank;
    for (int l = 0; l < nmats; ++l) {
        if (rows[l] < 1 || cols[l] < 1) return GQ_ERR_ARG;
        s.total += (long long)rows[l] * cols[l];
        s.ptotal += (long long)rows[l] * rank;
        s.qtotal += (long long)cols[l] * rank;
        if (cols[l] % 4) s.vec = false;
        if (rows[l] > s.max_rows) s.max_rows = rows[l];
    }
    const int ct = s.vec ? 1024 : 256;
    int chunk = 4096;
    auto tiles = [&](int ch) {
        long long t = 0;
        for (int l = 0; l < nmats; ++l)
            t += (long long)W * ((cols[l] + ct - 1) / ct) * ((rows[l] + ch - 1) / ch);
        return t;
    };
    while (chunk > 128 && tiles(chunk) < kBackTargetTiles) chunk >>= 1;
    s.chunk_rows = chunk;
    s.chunks_max = (s.max_rows + chunk - 1) / chunk;
    return GQ_OK;
}

// Workspace of the whole step: header, then each region 256-byte aligned.
struct PsgdWs {
    size_t pw, codes_p, max_p, qpart, qw, codes_q, max_q, qsum, end;
};

size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

PsgdWs psgd_ws(const PsgdShape& s) {
    PsgdWs o;
    size_t at = kWorkspaceHeader;
    o.pw = at;
    at = up256(at + (size_t)s.W * s.ptotal * sizeof(float));
    o.codes_p = at;
    at = up256(at + (size_t)s.W * s.ptotal);
    o.max_p = at;
    at = up256(at + (size_t)s.W * s.nmats * sizeof(float));
    o.qpart = at;
    at = up256(at + (size_t)s.chunks_max * s.W * s.qtotal * sizeof(float));
    o.qw = at;
    at = up256(at + (size_t)s.W * s.qtotal * sizeof(float));
    o.codes_q = at;
    at = up256(at + (size_t)s.W * s.qtotal);
    o.max_q = at;
    at = up256(at + (size_t)s.W * s.nmats * sizeof(float));
    o.qsum = at;
    at = up256(at + (size_t)s.qtotal * sizeof(float));
    o.end = at;
    return o;
}

enum class PsgdTiles { Project, Back, Reduce, Reconstruct, ReconstructCols };

// Fill the matrices l0 .. l0 + count - 1 and their work-tile prefix.
void psgd_group(PsgdArgs& a, const PsgdShape& s, int l0, int count, PsgdTiles kind) {
    long long goff = 0, poff = 0, qoff = 0;
    for (int l = 0; l < l0; ++l) {
        goff += (long long)s.rows[l] * s.cols[l];
        poff += (long long)s.rows[l] * s.rank;
        qoff += (long long)s.cols[l] * s.rank;
    }
    a.count = count;
    a.tile0[0] = 0;
    for (int i = 0; i < count; ++i) {
        const int n = s.rows[l0 + i], m = s.cols[l0 + i];
        a.rows[i] = n;
        a.cols[i] = m;
        a.goff[i] = goff;
        a.poff[i] = poff;
        a.qoff[i] = qoff;
        goff += (long long)n * m;
        poff += (long long)n * s.rank;
        qoff += (long long)m * s.rank;
        long long tiles = 0;
        switch (kind) {
            case PsgdTiles::Project: tiles = (long long)s.W * ((n + 15) / 16); break;
            case PsgdTiles::Back: {
                const int ct = s.vec ? 1024 : 256;
                tiles = (long long)s.W * ((m + ct - 1) / ct) *
                        ((n + s.chunk_rows - 1) / s.chunk_rows);
                break;
            }
            case PsgdTiles::Reduce:
                tiles = (long long)s.W * (((long long)m * s.rank + 255) / 256);
                break;
            case PsgdTiles::Reconstruct: tiles = (n + 7) / 8; break;
            case PsgdTiles::ReconstructCols:
                tiles = (long long)((m + 1023) / 1024) * ((n + 127) / 128);
                break;
        }
        a.tile0[i + 1] = a.tile0[i] + tiles;
    }
}

void psgd_common(PsgdArgs& a, const PsgdShape& s) {
    std::memset(&a, 0, sizeof(a));
    a.total = s.total;
    a.ptotal = s.ptotal;
    a.qtotal = s.qtotal;
    a.W = s.W;
    a.rank = s.rank;
    a.chunk_rows = s.chunk_rows;
}

}  // namespace

GQ_API int gq_psgd_workspace_bytes(int W, int nmats, const int* rows_host, const int* cols_host,
                                   int rank, size_t* bytes) {
    if (!bytes) return GQ_ERR_ARG;
    PsgdShape s;
    int rc = psgd_shape(W, nmats, rows_host, cols_host, rank, s);
    if (rc) return rc;
    *bytes = psgd_ws(s).end;
    return GQ_OK;
}

GQ_API int gq_psgd_project(const float* g_dev, float* m_dev, int W, int nmats,
                           const int* rows_host, const int* cols_host, int rank, int have_prev,
                           const float* p_prev_dev, const float* q_dev, float* pw_dev,
                           cudaStream_t stream) {
    const NvtxRange nvtx_range("gq_psgd_project");
    PsgdShape s;
    int rc = psgd_shape(W, nmats, rows_host, cols_host, rank, s);
    if (rc) return rc;
    if (!g_dev || !m_dev || !q_dev || !pw_dev || (have_prev && !p_prev_dev)) return GQ_ERR_ARG;
    if (!aligned16(g_dev) || !aligned16(m_dev) || !aligned16(q_dev) || !aligned16(pw_dev) ||
        (have_prev && !aligned16(p_prev_dev)))
        return GQ_ERR_ALIGN;
    PsgdArgs a;
    psgd_common(a, s);
    a.g = g_dev;
    a.m = m_dev;
    a.p = have_prev ? p_prev_dev : nullptr;
    a.q = q_dev;
    a.pw = pw_dev;
    a.have_prev = have_prev ? 1 : 0;
    for (int l0 = 0; l0 < nmats; l0 += kPsgdGroup) {
        const int count = nmats - l0 < kPsgdGroup ? nmats - l0 : kPsgdGroup;
        psgd_group(a, s, l0, count, PsgdTiles::Project);
        if ((rc = cuda_status(launch_psgd_project(a, s.vec, sm_count(), stream)))) return rc;
    }
    return GQ_OK;
}

GQ_API int gq_psgd_orthonormalize(float* p_dev, int nmats, const int* rows_host, int rank,
                                  cudaStream_t stream) {
    const NvtxRange nvtx_range("gq_psgd_orthonormalize");
    if (!rows_host || nmats < 1 || nmats > 4096) return GQ_ERR_ARG;
    // only the row counts matter here; the column counts are set to a valid
    // placeholder so that the shared shape check and offsets apply
    const std::vector<int> any_cols((size_t)nmats, 4);
    PsgdShape s;
    int rc = psgd_shape(1, nmats, rows_host, any_cols.data(), rank, s);
    if (rc) return rc;
    if (!p_dev) return GQ_ERR_ARG;
    if (!aligned16(p_dev)) return GQ_ERR_ALIGN;
    PsgdArgs a;
    psgd_common(a, s);
    a.psum = p_dev;
    for (int l0 = 0; l0 < nmats; l0 += kPsgdGroup) {
        const int count = nmats - l0 < kPsgdGroup ? nmats - l0 : kPsgdGroup;
        psgd_group(a, s, l0, count, PsgdTiles::Project);
        if ((rc = cuda_status(launch_psgd_orth(a, stream)))) return rc;
    }
    return GQ_OK;
}

GQ_API int gq_psgd_back_project(const float* m_dev, const float* p_dev, int W, int nmats,
                                const int* rows_host, const int* cols_host, int rank,
                                float* qw_dev, void* ws_dev, cudaStream_t stream) {
    const NvtxRange nvtx_range("gq_psgd_back_project");
    PsgdShape s;
    int rc = psgd_shape(W, nmats, rows_host, cols_host, rank, s);
    if (rc) return rc;
    if (!m_dev || !p_dev || !qw_dev || !ws_dev) return GQ_ERR_ARG;
    if (!aligned16(m_dev) || !aligned16(p_dev) || !aligned16(qw_dev) || !aligned16(ws_dev))
        return GQ_ERR_ALIGN;
    const PsgdWs o = psgd_ws(s);
    PsgdArgs a;
    psgd_common(a, s);
    a.m = const_cast<float*>(m_dev);
    a.p = p_dev;
    a.qpart = reinterpret_cast<float*>(static_cast<char*>(ws_dev) + o.qpart);
    a.qw = qw_dev;
    for (int l0 = 0; l0 < nmats; l0 += kPsgdGroup) {
        const int count = nmats - l0 < kPsgdGroup ? nmats - l0 : kPsgdGroup;
        psgd_group(a, s, l0, count, PsgdTiles::Back);
        if ((rc = cuda_status(launch_psgd_back(a, s.vec, sm_count(), stream)))) return rc;
        psgd_group(a, s, l0, count, PsgdTiles::Reduce);
        if ((rc = cuda_status(launch_psgd_back_reduce(a, sm_count(), stream)))) return rc;
    }
    return GQ_OK;
}

GQ_API int gq_psgd_mean(const float* sum_dev, float* out_dev, long long n, int W,
                        cudaStream_t stream) {
    const NvtxRange nvtx_range("gq_psgd_mean");
    if (!sum_dev || !out_dev || n < 0 || W < 1) return GQ_ERR_ARG;
    if (!aligned4(sum_dev) || !aligned4(out_dev)) return GQ_ERR_ALIGN;
    if (n == 0) return GQ_OK;
    return cuda_status(launch_psgd_mean(sum_dev, out_dev, n, W, sm_count(), stream));
}

GQ_API int gq_psgd_reconstruct(const float* p_dev, const float* q_dev, int nmats,
                               const int* rows_host, const int* cols_host, int rank,
                               float* ghat_dev, cudaStream_t stream) {
    const NvtxRange nvtx_range("gq_psgd_reconstruct");
    PsgdShape s;
    int rc = psgd_shape(1, nmats, rows_host, cols_host, rank, s);
    if (rc) return rc;
    if (!p_dev || !q_dev || !ghat_dev) return GQ_ERR_ARG;
    if (!aligned16(p_dev) || !aligned16(q_dev) || !aligned16(ghat_dev)) return GQ_ERR_ALIGN;
    PsgdArgs a;
    psgd_common(a, s);
    a.p = p_dev;
    a.q = q_dev;
    a.out = ghat_dev;
    for (int l0 = 0; l0 < nmats; l0 += kPsgdGroup) {
        const int count = nmats - l0 < kPsgdGroup ? nmats - l0 : kPsgdGroup;
        if (s.vec) {
            psgd_group(a, s, l0, count, PsgdTiles::ReconstructCols);
            rc = cuda_status(launch_psgd_reconstruct_cols(a, sm_count(), stream));
        } else {
            psgd_group(a, s, l0, count, PsgdTiles::Reconstruct);
            rc = cuda_status(launch_psgd_reconstruct(a, s.vec, sm_count(), stream));
        }
        if (rc) return rc;
    }
    return GQ_OK;
}

GQ_API int gq_lqsgd_step(const float* g_dev, float* m_dev, int W, int nmats,
                         const int* rows_host, const int* cols_host, int rank, int have_prev,
                         const gq_config* cfg, float* p_dev, float* q_dev, float* ghat_dev,
                         void* ws_dev, cudaStream_t stream) {
    const NvtxRange nvtx_range("gq_lqsgd_step");
    if (!cfg || cfg->levels != GQ_LOG || !(cfg->alpha > 0.f) || !(cfg->alpha <= 3.0e38f))
        return GQ_ERR_ARG;
    // the step derives two streams (2t, 2t + 1) on the host: no device step word
    if (cfg->step_dev) return GQ_ERR_ARG;
    PsgdShape s;
    int rc = psgd_shape(W, nmats, rows_host, cols_host, rank, s);
    if (rc) return rc;
    if (!g_dev || !m_dev || !p_dev || !q_dev || !ws_dev) return GQ_ERR_ARG;
    if (!aligned16(g_dev) || !aligned16(m_dev) || !aligned16(p_dev) || !aligned16(q_dev) ||
        !aligned16(ws_dev) || (ghat_dev && !aligned16(ghat_dev)))
        return GQ_ERR_ALIGN;
    const PsgdWs o = psgd_ws(s);
    char* ws = static_cast<char*>(ws_dev);
    float* pw = reinterpret_cast<float*>(ws + o.pw);
    float* qw = reinterpret_cast<float*>(ws + o.qw);
    float* qsum = reinterpret_cast<float*>(ws + o.qsum);
    signed char* codes_p = reinterpret_cast<signed char*>(ws + o.codes_p);
    signed char* codes_q = reinterpret_cast<signed char*>(ws + o.codes_q);
    float* max_p = reinterpret_cast<float*>(ws + o.max_p);
    float* max_q = reinterpret_cast<float*>(ws + o.max_q);
    std::vector<int> ranks((size_t)nmats, rank);
    gq_config c = *cfg;
    // P_w = M_w Q (with the deferred error), then its log-quantized sum
    rc = gq_psgd_project(g_dev, m_dev, W, nmats, rows_host, cols_host, rank, have_prev, p_dev,
                         q_dev, pw, stream);
    if (rc) return rc;
    c.step = 2u * cfg->step;
    rc = gq_logq_quantize(pw, W, nmats, rows_host, ranks.data(), &c, max_p, codes_p, ws_dev,
                          stream);
    if (rc) return rc;
    rc = gq_logq_decode_sum(codes_p, max_p, W, nmats, rows_host, ranks.data(), &c, p_dev, stream);
    if (rc) return rc;
    rc = gq_psgd_orthonormalize(p_dev, nmats, rows_host, rank, stream);
    if (rc) return rc;
    // Q_w = M_w^T P_hat, its log-quantized sum, and the mean
    rc = gq_psgd_back_project(m_dev, p_dev, W, nmats, rows_host, cols_host, rank, qw, ws_dev,
                              stream);
    if (rc) return rc;
    c.step = 2u * cfg->step + 1u;
    rc = gq_logq_quantize(qw, W, nmats, cols_host, ranks.data(), &c, max_q, codes_q, ws_dev,
                          stream);
    if (rc) return rc;
    rc = gq_logq_decode_sum(codes_q, max_q, W, nmats, cols_host, ranks.data(), &c, qsum, stream);
    if (rc) return rc;
    rc = gq_psgd_mean(qsum, q_dev, s.qtotal, W, stream);
    if (rc) return rc;
    if (ghat_dev)
        rc = gq_psgd_reconstruct(p_dev, q_dev, nmats, rows_host, cols_host, rank, ghat_dev, stream);
    return rc;
}

}  // extern "C"
