// Programmatic dependent launch for the layer-gather kernels. A stage-3 walk
// is a chain of short copy kernels on one stream (one per layer unit, each a
// few tens of microseconds); with an ordinary launch the GPU idles between
// them while the next grid is launched. A kernel launched with launch_pdl may
// be scheduled while the previous kernel on the stream is still finishing; it
// calls pdl_wait() before its first global-memory access, which returns once
// that kernel has completed and its writes are visible, so the ordering is
// the same as with an ordinary launch. pdl_launch_dependents() lets the next
// such kernel be scheduled as this one's blocks retire. Internal to libzero.
#pragma once

#include <cuda_runtime.h>

#include <utility>

namespace zk {

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args)
{
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace zk
