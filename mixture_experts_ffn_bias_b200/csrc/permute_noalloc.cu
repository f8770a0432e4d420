// moe_permute for callers that cannot allocate device memory.
//
// moe_permute takes its scratch (per-block expert counts and a status word)
// from a caller workspace.  Some callers have no way to provide one: a plain
// C host program that links only this library and has no device allocator of
// its own, or a serving loop that runs on a fixed memory plan and must not
// call cudaMalloc/cudaFree after start-up (those calls synchronise the whole
// device and can fail once memory is fragmented).  This variant keeps its
// scratch in a fixed array in the library's own device memory instead.
//
// The array below exists once per GPU that loads the library and stays
// allocated until the process exits.  Its name is only a host-side stand-in
// in host code, so the device address is looked up with
// cudaGetSymbolAddress, once per device, with that device current.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/moe.h"
#include "kernels.h"

namespace {

// Scratch ints: [0] status word, [64, 64 + kNoAllocBlkInts) per-block counts
// (256-byte aligned start).  1 MiB + 256 B per device.
constexpr int kNoAllocHeadInts = 64;
constexpr int kNoAllocBlkInts = MOE_PERMUTE_NOALLOC_MAX_BLOCK_COUNTS;

static __device__ __align__(256) int32_t g_permute_scratch[kNoAllocHeadInts + kNoAllocBlkInts];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
int32_t* g_scratch_ptr[kMaxDevices] = {};

// Device address of this device's copy of the scratch array; set up on the
// first call per device.
moe_status scratch_for_current_device(int32_t** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess || p == nullptr)
      return MOE_ERR_CUDA;
    g_scratch_ptr[dev] = static_cast<int32_t*>(p);
  }
  *out = g_scratch_ptr[dev];
  return MOE_OK;
}

inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool al4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

}  // namespace

extern "C" moe_status moe_permute_noalloc(const moe_config* cfg, const int32_t* topk_idx,
                                          const void* x, int32_t* counts, int32_t* offsets,
                                          int32_t* slot_pos, int32_t* perm_src, void* x_perm,
                                          void* stream) {
  moe_status st = moe_check_config(cfg);
  if (st != MOE_OK) return st;
  if (!counts || !offsets || !al4(counts) || !al4(offsets)) return MOE_ERR_INVALID;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cfg->T == 0) {
    if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * cfg->n_experts, s) != cudaSuccess ||
        cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (cfg->n_experts + 1), s) != cudaSuccess)
      return MOE_ERR_CUDA;
    return MOE_OK;
  }
  if (!topk_idx || !x || !slot_pos || !perm_src || !x_perm) return MOE_ERR_INVALID;
  if (!al16(x) || !al16(x_perm) || !al4(topk_idx) || !al4(slot_pos) || !al4(perm_src))
    return MOE_ERR_INVALID;
  const int nblk = moe::rank_blocks(cfg->T);
  if (static_cast<long long>(nblk) * cfg->n_experts > kNoAllocBlkInts)
    return MOE_ERR_WORKSPACE;   // the fixed scratch cannot hold this T x E
  int32_t* scratch = nullptr;
  if ((st = scratch_for_current_device(&scratch)) != MOE_OK) return st;
  uint32_t* status = reinterpret_cast<uint32_t*>(scratch);
  int32_t* blk = scratch + kNoAllocHeadInts;
  // The status word must start at zero; every block count the scan reads is
  // written by the rank kernel of the same call.
  if (cudaMemsetAsync(status, 0, sizeof(uint32_t), s) != cudaSuccess) return MOE_ERR_CUDA;
  if (moe::dispatch_rank(topk_idx, cfg->T, cfg->top_k, cfg->n_experts, blk, slot_pos, status,
                         s) != cudaSuccess ||
      moe::dispatch_scan(blk, nblk, cfg->n_experts, counts, offsets, s) != cudaSuccess ||
      moe::dispatch_scatter(cfg->dtype == MOE_BF16, x, topk_idx, blk, slot_pos, perm_src, x_perm,
                            cfg->T, cfg->d_model, cfg->top_k, cfg->n_experts, moe::kRankBlock,
                            s) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}
