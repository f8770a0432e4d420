// Dispatch: token-to-expert histogram, prefix scan and the stable permutation
// of the T*k routed pairs into expert-contiguous rows (the row order grouped_mm
// dispatch consumes; SpecForge PR #930 "Why FSDP is enough here", PR #931
// "What works": grouped GEMM checked against a sorted loop over experts).
//
// The row of pair (t, j) that chose expert e is
//     offsets[e] + #{t' < t : token t' chose e},
// i.e. the pairs are stably sorted by (expert, token).  Three kernels, no
// global atomics, deterministic:
//   rank     per block of 256 tokens: a 256-bit token mask per expert in
//            shared memory; a pair's rank inside its block is a popcount of
//            the mask bits of earlier tokens; the popcount of the whole mask
//            is the block's count for that expert.
//   scan     one block: per expert, running sums over blocks (block bases);
//            exclusive scan over experts (offsets).
//   scatter  one warp per token: final row = base + rank, x row read once
//            and written to its k rows with 16-byte vector accesses.
// Pairs with an expert id outside [0, E), or repeating an expert the token
// already chose, are skipped (row -1) and flagged in the status word.
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.h"
#include "launch.cuh"
#include "sm100.cuh"

namespace moe {
namespace {

constexpr int kMaxE = 256;
constexpr int kWords = kRankBlock / 32;

__device__ __forceinline__ bool pair_valid(const int32_t* __restrict__ row, int j, int E) {
  const int e = row[j];
  if (e < 0 || e >= E) return false;
  for (int jj = 0; jj < j; ++jj)
    if (row[jj] == e) return false;
  return true;
}

__global__ void __launch_bounds__(kRankBlock)
dispatch_rank_kernel(const int32_t* __restrict__ topk_idx, int T, int k, int E,
                     int32_t* __restrict__ blk_counts, int32_t* __restrict__ rank_out,
                     uint32_t* __restrict__ status) {
  pdl_trigger();
  pdl_wait();
  __shared__ uint32_t masks[kMaxE][kWords];
  const int tid = threadIdx.x;
  const int lane = tid & 31, word = tid >> 5;
  const int t = blockIdx.x * kRankBlock + tid;
  for (int i = tid; i < E * kWords; i += kRankBlock) masks[i / kWords][i % kWords] = 0u;
  __syncthreads();
  const int32_t* row = topk_idx + static_cast<size_t>(t) * k;
  bool bad = false;
  if (t < T) {
    for (int j = 0; j < k; ++j) {
      if (pair_valid(row, j, E))
        atomicOr(&masks[row[j]][word], 1u << lane);
      else
        bad = true;
    }
  }
  __syncthreads();
  if (t < T) {
    const uint32_t below = (1u << lane) - 1u;
    for (int j = 0; j < k; ++j) {
      int r = -1;
      if (pair_valid(row, j, E)) {
        const int e = row[j];
        r = __popc(masks[e][word] & below);
        for (int w = 0; w < word; ++w) r += __popc(masks[e][w]);
      }
      rank_out[static_cast<size_t>(t) * k + j] = r;
    }
  }
  if (bad) atomicOr(status, kDevBadIndex);
  for (int e = tid; e < E; e += kRankBlock) {
    int c = 0;
#pragma unroll
    for (int w = 0; w < kWords; ++w) c += __popc(masks[e][w]);
    blk_counts[static_cast<size_t>(blockIdx.x) * E + e] = c;
  }
}

// The rank kernel with the scan folded in: each block, once its counts are
// out, takes a ticket; the last block to finish turns all block counts into
// block bases, counts and offsets (the same arithmetic as the scan kernel
// below), then puts the ticket counter back to zero.  done: zero at launch.
// fold_cnt (or null): the folded combine's per-(token, column tile) counts,
// set to the number of the token's skipped pairs (rows that never arrive).
__global__ void __launch_bounds__(kRankBlock)
dispatch_rank_scan_kernel(const int32_t* __restrict__ topk_idx, int T, int k, int E,
                          int32_t* __restrict__ blk, int32_t* __restrict__ rank_out,
                          int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                          uint32_t* __restrict__ status, uint32_t* __restrict__ done,
                          int32_t* __restrict__ fold_cnt, int fold_nt) {
  pdl_trigger();
  pdl_wait();
  __shared__ uint32_t masks[kMaxE][kWords];
  __shared__ int s_last;
  const int tid = threadIdx.x;
  const int lane = tid & 31, word = tid >> 5;
  const int t = blockIdx.x * kRankBlock + tid;
  for (int i = tid; i < E * kWords; i += kRankBlock) masks[i / kWords][i % kWords] = 0u;
  __syncthreads();
  const int32_t* row = topk_idx + static_cast<size_t>(t) * k;
  bool bad = false;
  if (t < T) {
    for (int j = 0; j < k; ++j) {
      if (pair_valid(row, j, E))
        atomicOr(&masks[row[j]][word], 1u << lane);
      else
        bad = true;
    }
  }
  __syncthreads();
  if (t < T) {
    const uint32_t below = (1u << lane) - 1u;
    for (int j = 0; j < k; ++j) {
      int r = -1;
      if (pair_valid(row, j, E)) {
        const int e = row[j];
        r = __popc(masks[e][word] & below);
        for (int w = 0; w < word; ++w) r += __popc(masks[e][w]);
      }
      rank_out[static_cast<size_t>(t) * k + j] = r;
    }
  }
  if (bad) atomicOr(status, kDevBadIndex);
  if (fold_cnt != nullptr && t < T) {
    int skipped = 0;
    for (int j = 0; j < k; ++j) skipped += pair_valid(row, j, E) ? 0 : 1;
    for (int c = 0; c < fold_nt; ++c) fold_cnt[static_cast<size_t>(t) * fold_nt + c] = skipped;
  }
  for (int e = tid; e < E; e += kRankBlock) {
    int c = 0;
#pragma unroll
    for (int w = 0; w < kWords; ++w) c += __popc(masks[e][w]);
    blk[static_cast<size_t>(blockIdx.x) * E + e] = c;
  }
  __threadfence();   // this block's counts are visible before its ticket
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(done, 1u) == gridDim.x - 1 ? 1 : 0;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // the scan: thread e walks expert e's column of block counts (read from
  // L2, sixteen loads in flight), then a block scan over the experts
  const int nblk = gridDim.x;
  int* s = reinterpret_cast<int*>(masks);   // kMaxE ints of the mask space
  const int e = tid;
  int run = 0;
  if (e < E) {
    for (int b0 = 0; b0 < nblk; b0 += 16) {
      int c[16];
#pragma unroll
      for (int u = 0; u < 16; ++u)
        c[u] = b0 + u < nblk ? __ldcg(blk + static_cast<size_t>(b0 + u) * E + e) : 0;
#pragma unroll
      for (int u = 0; u < 16; ++u) run += c[u];
    }
    counts[e] = run;
  }
  s[e] = e < E ? run : 0;
  __syncthreads();
  for (int o = 1; o < kMaxE; o <<= 1) {          // inclusive Hillis-Steele scan
    const int v = (e >= o) ? s[e - o] : 0;
    __syncthreads();
    s[e] += v;
    __syncthreads();
  }
  const int excl = s[e] - (e < E ? run : 0);
  if (e < E) offsets[e] = excl;
  if (e == kMaxE - 1) offsets[E] = s[e];
  if (e < E) {
    int base = excl;
    for (int b0 = 0; b0 < nblk; b0 += 16) {
      int c[16];
#pragma unroll
      for (int u = 0; u < 16; ++u)
        c[u] = b0 + u < nblk ? __ldcg(blk + static_cast<size_t>(b0 + u) * E + e) : 0;
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        if (b0 + u < nblk) blk[static_cast<size_t>(b0 + u) * E + e] = base;
        base += c[u];
      }
    }
  }
  if (tid == 0) *done = 0u;
}

// Block counts [nblk, E] -> block bases (in place), counts and offsets.  The
// counts are staged in shared memory when they fit (kScanSmemInts), so the
// per-expert running sums walk shared memory instead of global memory.
constexpr int kScanSmemInts = 11776;   // 46 KB + the 1 KB scan array stay under 48 KB

__global__ void __launch_bounds__(kMaxE)
dispatch_scan_kernel(int32_t* __restrict__ blk, int nblk, int E, int32_t* __restrict__ counts,
                     int32_t* __restrict__ offsets) {
  pdl_trigger();
  pdl_wait();
  __shared__ int s[kMaxE];
  __shared__ int sblk[kScanSmemInts];
  const int e = threadIdx.x;
  const int n = nblk * E;
  const bool staged = n <= kScanSmemInts;
  int32_t* col = staged ? sblk : blk;
  if (staged) {
    for (int i = threadIdx.x; i < n; i += blockDim.x) sblk[i] = blk[i];
    __syncthreads();
  }
  int run = 0;
  if (e < E) {
#pragma unroll 8
    for (int b = 0; b < nblk; ++b) {
      const int c = col[static_cast<size_t>(b) * E + e];
      col[static_cast<size_t>(b) * E + e] = run;
      run += c;
    }
    counts[e] = run;
  }
  s[e] = (e < E) ? run : 0;
  __syncthreads();
  for (int o = 1; o < kMaxE; o <<= 1) {          // inclusive Hillis-Steele scan
    const int v = (e >= o) ? s[e - o] : 0;
    __syncthreads();
    s[e] += v;
    __syncthreads();
  }
  const int excl = s[e] - ((e < E) ? run : 0);
  if (e < E) offsets[e] = excl;
  if (e == kMaxE - 1) offsets[E] = s[e];
  if (staged) {
    s[e] = excl;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) blk[i] = sblk[i] + s[i % E];
  } else if (e < E) {
#pragma unroll 8
    for (int b = 0; b < nblk; ++b) blk[static_cast<size_t>(b) * E + e] += excl;
  }
}

// One warp per token; `vecs` 16-byte vectors per row.
__global__ void __launch_bounds__(256)
dispatch_scatter_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ topk_idx,
                        const int32_t* __restrict__ bases, int32_t* __restrict__ slot_pos,
                        int32_t* __restrict__ perm_src, uint4* __restrict__ x_perm, int T,
                        int vecs, int k, int E, int blk_tokens) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  int my_slot = -1;
  if (lane < k) {
    const size_t p = static_cast<size_t>(t) * k + lane;
    const int r = slot_pos[p];
    if (r >= 0) {
      const int e = topk_idx[p];
      my_slot = bases[static_cast<size_t>(t / blk_tokens) * E + e] + r;
      perm_src[my_slot] = t;
    }
    slot_pos[p] = my_slot;
  }
  const uint4* src = x + static_cast<size_t>(t) * vecs;
  for (int c0 = lane; c0 < vecs; c0 += 32 * 4) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int c = c0 + 32 * u;
      if (c < vecs) v[u] = __ldcs(src + c);   // last use of x: evict first
    }
    for (int j = 0; j < k; ++j) {
      const int s = __shfl_sync(0xffffffffu, my_slot, j);
      if (s < 0) continue;
      uint4* dst = x_perm + static_cast<size_t>(s) * vecs;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = c0 + 32 * u;
        if (c < vecs) dst[c] = v[u];
      }
    }
  }
}

// One thread per token: final rows and the token of each row, no copy;
// zero[0, n_zero) set to zero on the way.
__global__ void __launch_bounds__(256)
dispatch_positions_kernel(const int32_t* __restrict__ topk_idx, const int32_t* __restrict__ bases,
                          int32_t* __restrict__ slot_pos, int32_t* __restrict__ perm_src, int T,
                          int k, int E, int blk_tokens, int32_t* __restrict__ zero, int n_zero) {
  pdl_trigger();
  pdl_wait();
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  for (int i = t; i < n_zero; i += gridDim.x * blockDim.x) zero[i] = 0;
  if (t >= T) return;
  const int32_t* b = bases + static_cast<size_t>(t / blk_tokens) * E;
  for (int j = 0; j < k; ++j) {
    const size_t p = static_cast<size_t>(t) * k + j;
    const int r = slot_pos[p];
    int slot = -1;
    if (r >= 0) {
      slot = b[topk_idx[p]] + r;
      perm_src[slot] = t;
    }
    slot_pos[p] = slot;
  }
}

}  // namespace

cudaError_t dispatch_positions(const int32_t* topk_idx, const int32_t* blk_bases,
                               int32_t* slot_pos, int32_t* perm_src, int T, int k, int E,
                               int blk_tokens, cudaStream_t stream, int32_t* zero, int n_zero) {
  return launch_pdl(dispatch_positions_kernel, dim3((T + 255) / 256), dim3(256), 0, stream,
                    topk_idx, blk_bases, slot_pos, perm_src, T, k, E, blk_tokens, zero,
                    zero != nullptr ? n_zero : 0);
}

cudaError_t dispatch_rank(const int32_t* topk_idx, int T, int k, int E, int32_t* blk_counts,
                          int32_t* rank_out, uint32_t* status, cudaStream_t stream) {
  return launch_pdl(dispatch_rank_kernel, dim3(rank_blocks(T)), dim3(kRankBlock), 0, stream,
                    topk_idx, T, k, E, blk_counts, rank_out, status);
}

cudaError_t dispatch_rank_scan(const int32_t* topk_idx, int T, int k, int E, int32_t* blk,
                               int32_t* rank_out, int32_t* counts, int32_t* offsets,
                               uint32_t* status, uint32_t* done, cudaStream_t stream,
                               int32_t* fold_cnt, int fold_nt) {
  if (E > kMaxE || kRankBlock != kMaxE) return cudaErrorInvalidValue;
  return launch_pdl(dispatch_rank_scan_kernel, dim3(rank_blocks(T)), dim3(kRankBlock), 0, stream,
                    topk_idx, T, k, E, blk, rank_out, counts, offsets, status, done, fold_cnt,
                    fold_nt);
}

cudaError_t dispatch_scan(int32_t* blk_counts, int nblk, int E, int32_t* counts,
                          int32_t* offsets, cudaStream_t stream) {
  return launch_pdl(dispatch_scan_kernel, dim3(1), dim3(kMaxE), 0, stream, blk_counts, nblk, E,
                    counts, offsets);
}

cudaError_t dispatch_scatter(bool bf16, const void* x, const int32_t* topk_idx,
                             const int32_t* blk_bases, int32_t* slot_pos, int32_t* perm_src,
                             void* x_perm, int T, int d, int k, int E, int blk_tokens,
                             cudaStream_t stream) {
  const int vecs = d * (bf16 ? 2 : 4) / 16;
  const int warps = 8;
  return launch_pdl(dispatch_scatter_kernel, dim3((T + warps - 1) / warps), dim3(warps * 32), 0,
                    stream, static_cast<const uint4*>(x), topk_idx, blk_bases, slot_pos, perm_src,
                    static_cast<uint4*>(x_perm), T, vecs, k, E, blk_tokens);
}

}  // namespace moe
