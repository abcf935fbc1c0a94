// gq_pdl.cuh -- programmatic dependent launch between the step's kernels
// (sm_90 and later; here sm_100a).
//
// A kernel launched with the programmatic-serialization attribute may be
// scheduled before the previous kernel in its stream has finished, once every
// block of that kernel has called pdl_launch_dependents (or exited).  It must
// call pdl_wait, which returns when the previous kernel has completed and its
// memory is visible, before it reads or writes any global memory the previous
// kernel may touch.  Both are no-ops for a kernel launched without the
// attribute.  The norm pass and the fused pass use it so that each one's
// launch and prologue overlap the tail of the kernel before it: measured with
// the L2 flushed between steps, a step of 4 x 2^20 coordinates took 23.6 us
// against 25.6 us, 8 x 2^18 17.4 against 20.4, 8 x 2^20 with error feedback
// 42.0 against 44.1, and from the ResNet-50 size (8 x 25.6 M) up no change;
// results are the same bit for bit.
#pragma once

#include <cuda_runtime.h>

#include <utility>

namespace gq {

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Whether launches on this stream take the attribute: not while the stream is
// being captured into a graph (the captured step keeps plain stream order).
inline bool pdl_allowed(cudaStream_t st) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    return cudaStreamIsCapturing(st, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusNone;
}

// cudaLaunchKernelEx with the programmatic-serialization attribute when pdl.
template <typename... KArgs, typename... Args>
cudaError_t launch_with_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                            cudaStream_t st, bool pdl, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

}  // namespace gq
