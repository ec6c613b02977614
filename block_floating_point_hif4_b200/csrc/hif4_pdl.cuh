// hif4_pdl.cuh — programmatic dependent launch for chains of dependent
// kernels on one stream.  A kernel of the chain calls pdl_enter() first: it
// waits for the previous grid (completion and memory) before its first
// global access, then lets the next grid launch, so only the launch and
// block set-up overlap.  Both instructions are no-ops for a normal launch.
#pragma once

#include <cuda_runtime.h>

#include "hif4_internal.cuh"

namespace hif4 {

__device__ __forceinline__ void pdl_enter()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
hif4_status launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...) != cudaSuccess) return HIF4_ERR_CUDA;
    return launch_status();
}

} // namespace hif4
