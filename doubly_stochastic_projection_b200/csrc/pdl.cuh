// pdl.cuh -- programmatic dependent launch for the short projection kernels.
//
// A kernel launched by launch_pdl may be scheduled while the kernel before it
// in the stream is still finishing, which hides the launch gap between two
// back-to-back kernels (a few microseconds, a sizeable part of a 131072-matrix
// projection).  Ordering is unchanged: such a kernel calls pdl_wait() before
// its first global memory access, and griddepcontrol.wait returns only once
// every grid it depends on has completed and its writes are visible.  A kernel
// then calls pdl_trigger() so that the next PDL launch in the stream may be
// scheduled; without a trigger that happens when the grid exits.  Both
// instructions are no-ops for a kernel launched the ordinary way.
#pragma once

#include <cuda_runtime.h>

namespace mhc {

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), int grid, int threads, size_t smem, cudaStream_t s,
                       Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3((unsigned)threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace mhc
