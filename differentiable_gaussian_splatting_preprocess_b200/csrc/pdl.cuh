// Programmatic dependent launch for the binning's chain of short kernels.
#pragma once

#include <cuda_runtime.h>

namespace gs {

// Programmatic dependent launch (sm_90 and later): a kernel launched with
// launch_pdl may be scheduled while the kernel before it in the stream is
// finishing; its threads first wait (griddepcontrol.wait: until that kernel
// has completed and its memory operations are visible).  No kernel triggers
// its dependents early, so the next grid is scheduled as this one's blocks
// exit: only the launch latency and the ramp-up overlap the previous
// kernel's tail, and no early-launched block holds an SM while it waits
// (measured: an early trigger cost graph replays more than it saved).  No
// kernel reads anything before its predecessor is complete.  Without the
// launch attribute the wait does nothing.
__device__ __forceinline__ void pdl_enter() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace gs
