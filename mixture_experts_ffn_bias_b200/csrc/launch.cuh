// Kernel launches with programmatic dependent launch (PDL).
//
// Every kernel of the library is launched with programmatic stream
// serialization: it may start while the previous kernel of the stream is
// finishing, runs its set-up (shared-memory and barrier initialisation, TMEM
// allocation, descriptor prefetch), and calls pdl_wait() before it touches
// any global memory a previous kernel may write; pdl_wait() returns once the
// previous grid has completed and its writes are visible.  Persistent
// kernels call pdl_trigger() when their producer has issued its last loads,
// which lets the next kernel's CTAs start on SMs that have gone idle.
// Launched without the attribute (or after a non-kernel operation) both are
// no-ops in effect.
#pragma once
#include <cuda_runtime.h>

#include <utility>

namespace moe {

__device__ __forceinline__ void pdl_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
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
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace moe
