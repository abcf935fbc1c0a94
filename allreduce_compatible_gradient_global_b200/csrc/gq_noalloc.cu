// gq_noalloc.cu -- gq_global_norm_noalloc: the global-scale reduction for
// callers that cannot allocate device memory, even a workspace.
//
// The ordinary gq_global_norm keeps its per-block partial sums and its
// last-block ticket in a workspace the caller allocates.  This variant keeps
// them in a file-scope __device__ array instead, so the caller passes only the
// gradients and the output buffers.  The array is small (kNoallocBytes) and
// every GPU that loads this library holds it until the process exits.
//
// Host code cannot use the array's name as a device address (on the host it
// is only a stand-in), so the first call on each device resolves the real
// address with cudaGetSymbolAddress, with that device current, and caches it.
// That first call should therefore come before any stream capture.  The
// cached address belongs to the device's context: after cudaDeviceReset the
// module is loaded again and the array may move, so this call must not be
// used across a device reset.
//
// The block count per worker row is gq_global_norm's own (the fp32 runs and
// the fp64 combine order depend on it), so the two calls return bit-identical
// scales and norms.  It always fits the array: 2 W nb <= 2 * 8 blocks per SM
// * the SM count, far below kNoallocSlots on any current GPU, and it is
// clamped to the array in any case.
#include <cuda_runtime.h>

#include <mutex>

#include "gq_api.h"
#include "gq_internal.h"

namespace {

constexpr int kNoallocSlots = 8192;       // fp64 partial slots (64 KiB)
constexpr int kNoallocMaxWorkers = 4096;  // W above this is rejected
constexpr int kNoallocMaxDevices = 64;
constexpr size_t kNoallocBytes =
    (size_t)gq::kWorkspaceHeader + (size_t)kNoallocSlots * sizeof(unsigned long long);

// Shared by every call on a device; the header (flag word, ticket counter) is
// cleared on the stream before each launch.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[kNoallocMaxDevices] = {};

// Device address of the scratch array on the current device (set-up on first use).
int scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GQ_ERR_CUDA;
    if (dev < 0 || dev >= kNoallocMaxDevices) return GQ_ERR_ARG;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_addr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
            return GQ_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return GQ_OK;
}

// Blocks per worker: those of gq_global_norm, within the array's partial
// slots (two per block).
int noalloc_blocks_per_worker(int W, long long d, int kind, bool has_e) {
    long long nb = gq::norm_blocks_per_worker(W, d, kind, has_e);
    if (nb > kNoallocSlots / (2 * W)) nb = kNoallocSlots / (2 * W);
    if (nb < 1) nb = 1;
    return (int)nb;
}

}  // namespace

extern "C" GQ_API int gq_global_norm_noalloc(const float* g_dev, const float* e_dev, int W,
                                             long long d, const gq_config* cfg, float* scale_dev,
                                             double* norms_dev, cudaStream_t stream) {
    if (!cfg || (!g_dev && d > 0) || !scale_dev) return GQ_ERR_ARG;
    if (W < 1 || d < 0) return GQ_ERR_ARG;
    if (W > kNoallocMaxWorkers) return GQ_ERR_SIZE;
    if (d > (1LL << 40) || (long long)W * d > (1LL << 42)) return GQ_ERR_ARG;
    if (cfg->scale_kind != GQ_SCALE_L2 && cfg->scale_kind != GQ_SCALE_MAXABS) return GQ_ERR_ARG;
    if (cfg->ef && !e_dev && d > 0) return GQ_ERR_ARG;
    const uintptr_t ga = reinterpret_cast<uintptr_t>(g_dev);
    const uintptr_t ea = reinterpret_cast<uintptr_t>(e_dev);
    if ((ga & 15u) || (cfg->ef && (ea & 15u)) || (reinterpret_cast<uintptr_t>(scale_dev) & 3u) ||
        (reinterpret_cast<uintptr_t>(norms_dev) & 7u))
        return GQ_ERR_ALIGN;
    void* scratch = nullptr;
    int rc = scratch_address(&scratch);
    if (rc) return rc;
    // the ticket counter must start at zero; the flag word is cleared with it
    if (cudaMemsetAsync(scratch, 0, (size_t)gq::kWorkspaceHeader, stream) != cudaSuccess)
        return GQ_ERR_CUDA;
    gq::NormArgs a;
    a.g = g_dev;
    a.e = cfg->ef ? e_dev : nullptr;
    a.d = d;
    a.W = W;
    a.nb = noalloc_blocks_per_worker(W, d, cfg->scale_kind, cfg->ef != 0);
    a.kind = cfg->scale_kind;
    a.scale = scale_dev;
    a.norms = norms_dev;
    a.partials = reinterpret_cast<unsigned long long*>(static_cast<char*>(scratch) +
                                                       gq::kWorkspaceHeader);
    a.hdr = reinterpret_cast<gq::WsHeader*>(scratch);
    return gq::launch_norm(a, (d % 4) == 0, stream) == cudaSuccess ? GQ_OK : GQ_ERR_CUDA;
}
