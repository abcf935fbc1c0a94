// gq_internal.h -- kernel argument blocks and launchers shared by the host
// entry points (gq_api.cu) and the kernel translation units.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "gq_device.cuh"

namespace gq {

constexpr int kThreads = 256;          // threads per block of every streaming kernel
constexpr int kMaxNormBlocks = 2048;   // norm blocks per worker (two 8-byte workspace slots each)
constexpr int kWorkspaceHeader = 256;  // flag word, ticket counter, padding

// Workspace header words.
struct WsHeader {
    unsigned int flags;    // bit 0: non-finite scale; bit 1: non-finite LQ max
    unsigned int counter;  // last-block ticket of the norm kernel (0 between calls)
    unsigned int tile_next;  // fused pass: next unclaimed tile (0 between calls)
    unsigned int tile_done;  // fused pass: producers finished (0 between calls)
};

constexpr unsigned kFlagNonfiniteScale = 1u;
constexpr unsigned kFlagNonfiniteLogqMax = 2u;
constexpr unsigned kFlagPipelineTimeout = 4u;  // a bounded mbarrier wait expired

struct NormArgs {
    const float* g;
    const float* e;
    long long d;
    int W;
    int nb;  // blocks per worker (gridDim.x)
    int kind;
    float* scale;
    double* norms;
    unsigned long long* partials;  // [W][nb]
    WsHeader* hdr;
};

struct QuantArgs {
    RoundKeys rk;
    const float* g;
    float* e;  // v = g + e is read when error feedback is on
    int update_e;  // 1: also write e <- v - Q(v) (step 5); 0: read only
    const float* scale;
    unsigned char* codes;  // [W][row_bytes] or null
    long long row_bytes;
    void* sum;  // [d] int8/int16 or null
    float* out; // [d] or null
    long long d;
    int W;
    int wire;  // bytes per sum element
    unsigned int step;
    unsigned int worker0;  // Philox worker index of row 0
    unsigned long long q0;  // coord0 / 4: Philox block counter of column 0
    const unsigned int* step_dev;  // non-null: the step is read here, not from `step`
    int L;
    float smax;        // (float)s
    float finest;      // 2^-(L-1)
    float inv_finest;  // 2^(L-1)
    float exp_shift;   // 2^(L-127): moves the finest level onto 2^-126
    float inv_w;       // 1/W when W is a power of two
    int w_pow2;
    WsHeader* hdr;  // flag word for pipeline timeouts
    // per-bucket scales (null: one global scale): the multiplier and unit of
    // 128-coordinate block b are bq_mult[b >> bucket_shift], bq_unit[...]
    const float* bq_mult;
    const float* bq_unit;
    int bucket_shift;
};

struct BucketArgs {
    const float* g;
    const float* e;
    long long d;
    long long nbuckets;
    long long nchunks;  // ceil(d / 2^chunk_log2)
    int W;
    int bucket_log2;  // bucket = 2^bucket_log2 coordinates, 7 <= bucket_log2 <= 30
    int chunk_log2;   // min(bucket_log2, 12)
    int kind;         // 0: L2, 1: max-abs
    int levels;       // 0: uniform, 1: exponential
    float smax;
    float finest;
    float* scales;  // [nbuckets] S_k
    float* mult;    // [nbuckets] multiplier of the fused pass
    float* unit;    // [nbuckets] value of one unit (decode / error feedback)
    double* part_sum;    // [W][nchunks] per-chunk sums of squares
    unsigned* part_max;  // [W][nchunks] per-chunk max |v| bits
    WsHeader* hdr;
};

struct AggArgs {
    const unsigned char* codes;
    long long row_bytes;
    void* sum;
    long long d;
    int W;
    int wire;
};

struct DequantArgs {
    const void* sum;  // null: no output decode
    const unsigned char* codes;
    long long row_bytes;
    const float* g;
    float* e;  // null: no error feedback
    const float* scale;
    float* out;
    long long d;
    int W;
    int wire;
    float smax;
    float finest;
    float inv_w;
    int w_pow2;
};

constexpr int kLogqGroup = 128;  // matrices per LQ launch (offsets ride in the parameters)

struct LogqArgs {
    const float* x;
    signed char* codes;
    float* maxabs;
    const signed char* ccodes;  // decode: input codes
    const float* cmaxabs;       // decode: input max-abs
    float* out;                 // decode: output sum
    long long total;            // elements per worker
    int W;
    int nmats;  // total matrices (row stride of maxabs)
    int m0;     // first matrix of this launch
    int count;  // matrices in this launch
    long long off[kLogqGroup + 1];
    unsigned int step;
    unsigned int worker0;  // Philox worker index of row 0
    const unsigned int* step_dev;  // non-null: the step is read here, not from `step`
    unsigned int seed_lo, seed_hi;
    float alpha;
    WsHeader* hdr;
};

// Raise a kernel's dynamic shared-memory limit only when a larger size is
// needed on this device: `limits` is the caller's per-kernel record (one
// static array per kernel instantiation).  Later calls, including calls made
// while a stream is being captured into a graph, then make no runtime call.
inline cudaError_t ensure_dynamic_smem(const void* kern, size_t smem, int* limits) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    if ((int)smem <= __atomic_load_n(&limits[dev], __ATOMIC_ACQUIRE)) return cudaSuccess;
    const cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess) __atomic_store_n(&limits[dev], (int)smem, __ATOMIC_RELEASE);
    return e;
}

// Launchers (return the cudaGetLastError() of the launch).
cudaError_t launch_norm(const NormArgs& a, bool vec, cudaStream_t st);
// Resident blocks per SM of the norm kernel instantiation for (kind, e?, vec).
int norm_resident_blocks(int kind, bool has_e, bool vec);
// Blocks per worker row of the norm kernel on the current device (its grid's x).
int norm_blocks_per_worker(int W, long long d, int kind, bool has_e);
cudaError_t launch_quant(const QuantArgs& a, int levels, int bits, bool ef, bool vec, int grid,
                         cudaStream_t st);
cudaError_t launch_aggregate(const AggArgs& a, int levels, int bits, int grid, cudaStream_t st);
cudaError_t launch_dequant(const DequantArgs& a, int levels, int bits, bool vec, int grid,
                           cudaStream_t st);
// The fused pass with the worker rows staged in shared memory by bulk copies
// (d % 4 == 0 and 16-byte-aligned rows only).
size_t tma_smem_bytes(int W, bool ef, int stages);
cudaError_t launch_quant_tma(const QuantArgs& a, int levels, int bits, bool ef, int stages,
                             int grid, cudaStream_t st);
// Bounded-wait self-test (raises kFlagPipelineTimeout after limit_ns).
cudaError_t launch_wait_timeout_selftest(WsHeader* hdr, unsigned long long limit_ns,
                                         cudaStream_t st);
cudaError_t launch_bucket_scales(const BucketArgs& a, int sms, cudaStream_t st);
cudaError_t launch_advance_step(unsigned int* step_dev, unsigned int by, cudaStream_t st);
cudaError_t launch_logq_quantize(const LogqArgs& a, cudaStream_t st);
cudaError_t launch_logq_decode(const LogqArgs& a, cudaStream_t st);

}  // namespace gq
