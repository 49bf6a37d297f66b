// Programmatic dependent launch.  A kernel launched with programmatic stream serialization may
// start before the previous kernel on its stream has finished (its CTAs take SMs as they free up);
// it calls pdl_wait before it touches anything the previous kernel writes, and returns from it once
// that kernel has completed and its memory operations are visible.  pdl_trigger lets the next such
// launch start before this one ends.  Both are no-ops in an ordinary launch.
#pragma once
#include <cuda_runtime.h>

namespace lsa {

__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// A launch configuration with programmatic stream serialization; attr holds the attribute.
inline cudaLaunchConfig_t pdl_config(dim3 grid, dim3 block, size_t smem, cudaStream_t st, cudaLaunchAttribute *attr)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cfg;
}

}  // namespace lsa
