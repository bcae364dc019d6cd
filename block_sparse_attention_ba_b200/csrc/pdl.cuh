// pdl.cuh — programmatic dependent launch (sm_90 and later) for kernel
// chains on one stream.
//
// A kernel launched with launch_dependent() may be scheduled before its
// predecessor in the stream has finished, as soon as every CTA of the
// predecessor has called pdl_allow_dependents() or exited, so that its
// launch and prologue overlap the predecessor's tail. It must call
// pdl_wait() before it reads what the predecessor writes or writes what the
// predecessor reads; pdl_wait() returns once the predecessor has completed
// and its memory operations are visible. Both are no-ops in a kernel that
// was launched normally.
#pragma once

#include <cuda_runtime.h>

namespace baatt {

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_allow_dependents() { asm volatile("griddepcontrol.launch_dependents;" :::); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                                    Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace baatt
