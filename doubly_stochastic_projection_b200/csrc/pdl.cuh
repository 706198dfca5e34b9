// pdl.cuh -- programmatic dependent launch for the short projection kernels.
//
// A kernel launched by launch_pdl may be scheduled while the kernel before it
// in the stream is finishing, which hides most of the launch gap between two
// back-to-back kernels (a sizeable part of a 131072-matrix projection).
// Ordering is unchanged: such a kernel calls pdl_wait() before its first
// global memory access, and griddepcontrol.wait returns only once every grid
// it depends on has completed and its writes are visible.
//
// The kernels do not execute griddepcontrol.launch_dependents, so a
// dependent grid is released when the primary grid exits.  Released at the
// start of the primary instead, the dependent's CTAs occupy the SMs while the
// primary still runs and wait there; measured on B200, back-to-back Newton
// forwards of 131072 matrices took 21.0 us a launch that way against 13.7 us
// released at exit (13.8 us without programmatic launch at all), and the
// forward + backward step 24.9 us against 19.7 us (20.8 us without).
#pragma once

#include <cuda_runtime.h>

namespace mhc {

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

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
