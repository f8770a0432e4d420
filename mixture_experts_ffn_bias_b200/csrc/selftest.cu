// Self-test of the bounded waits the tensor-core kernels use: a kernel waits
// on an mbarrier phase that nothing completes, gives up after a short limit,
// records kDevTimeout in the workspace status word and returns normally, so
// the context stays usable.  Nothing here faults, traps or hangs.
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/moe.h"
#include "kernels.h"
#include "sm100.cuh"

namespace {

__global__ void bounded_wait_selftest_kernel(uint32_t* status, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    moe::mbar_init(&bar, 1);      // one arrival expected; none will come
    abort_flag = 0;
    moe::fence_mbar_init();
  }
  __syncthreads();
  const bool ok = moe::mbar_wait(&bar, 0, &abort_flag, limit_ns);
  __syncthreads();
  if (threadIdx.x == 0 && (!ok || abort_flag)) atomicOr(status, moe::kDevTimeout);
}

}  // namespace

extern "C" moe_status moe_selftest_bounded_wait(void* ws, size_t ws_bytes, double limit_seconds,
                                                void* stream) {
  if (ws == nullptr || ws_bytes < 256 || (reinterpret_cast<uintptr_t>(ws) & 255u))
    return MOE_ERR_INVALID;
  if (!(limit_seconds > 0.0) || limit_seconds > 2.0) return MOE_ERR_INVALID;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t* status = static_cast<uint32_t*>(ws);
  if (cudaMemsetAsync(status, 0, sizeof(uint32_t), s) != cudaSuccess) return MOE_ERR_CUDA;
  bounded_wait_selftest_kernel<<<1, 32, 0, s>>>(
      status, static_cast<unsigned long long>(limit_seconds * 1e9));
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
