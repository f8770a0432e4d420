// Grouped GEMM over expert segments on 5th-generation tensor cores (tcgen05).
//
// For every group g (an expert, or the single shared-expert group) with rows
// [off[g], off[g+1]) of A:
//   SWIGLU pass (gate/up):  h[r, n] = silu(A[r] . W1[g][n]) * (A[r] . W3[g][n])
//   plain pass  (down):     y[r, n] = A[r] . W2[g][n]
// i.e. the two halves of the SwiGLU expert y = W2 (silu(W1 x) * (W3 x)) run
// over the expert-contiguous rows that grouped_mm dispatch consumes (SpecForge
// PR #930, "Why FSDP is enough here": compute scales with routed tokens, not
// with the number of experts; weights stacked [E, out, in]).
//
// One persistent kernel on CTA pairs (cluster of two, tcgen05.mma.cta_group::2,
// M = 256 rows per tile, static round-robin over tiles):
//   warp 0      TMA producer: per stage this CTA's 128 A rows x 64 K and its
//               half of the B tile, 128-byte swizzle, a ring of stages; A rows
//               may instead be gathered from x by the permutation
//               (tile::gather4, four rows per lane)
//   warp 1      allocates TMEM; on rank 0 one lane issues the MMAs for the
//               pair (bf16 x bf16 -> fp32) and commits stages / accumulators
//               to both CTAs
//   warps 2-5   epilogue: tcgen05.ld the accumulator (thread = row), SwiGLU
//               in fp32 (gate and up columns of an output column sit in the
//               same accumulator row: rank 0 holds the W1 rows of the B tile,
//               rank 1 the W3 rows), bf16 rounding, TMA tensor stores
// The TMEM accumulator is double buffered (up to 256 columns) so the
// epilogue of tile i overlaps the MMAs of tile i+1.  Tile order is (group,
// m-tile, n-tile) with n fastest, so CTAs running at the same time share the A
// tile and one expert's weights in L2.  The shared expert can run as one more
// group after the routed ones, with tensors of its own.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "kernels.h"
#include "launch.cuh"
#include "sm100.cuh"

namespace moe {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;                    // 64 bf16 = 128 bytes = one swizzle row
constexpr int A_STAGE_BYTES = BM * BK * 2;
constexpr int NUM_THREADS = 192;          // 6 warps
// A gate/up launch that fills its own A rows runs COPY_WARPS more warps.
constexpr int COPY_WARPS = 2;
constexpr int NUM_THREADS_COPY = NUM_THREADS + 32 * COPY_WARPS;

constexpr int MAX_GROUPS = 257;


// Variants of a mode, each its own instantiation, so the default path
// compiles without the alternatives' code:
//   VAR_NONE    A by TMA tiles, output by TMA stores
//   VAR_GATHER  (gate/up) A rows gathered from x by tile::gather4 loads
//   VAR_COPY    (gate/up) A rows copied into place by the launch itself
//   VAR_FOLD    (plain) the combine folded into the epilogue
constexpr int VAR_NONE = 0;
constexpr int VAR_GATHER = 1;
constexpr int VAR_COPY = 2;
constexpr int VAR_FOLD = 3;

// Epilogue / operand modes.
constexpr int MODE_PLAIN_BF16 = 0;    // C = A B^T, rounded to bf16
constexpr int MODE_SWIGLU_BF16 = 1;   // C = silu(A B0^T) * (A B1^T), rounded to bf16
// C = A B with B stored [K, N] per group (MN-major, N contiguous), rounded to
// bf16; the K rows of a group come from B0 (the first kb_split k-blocks) and
// then from B1, so [W1; W3] needs no concatenated copy.
constexpr int MODE_PLAIN_BMN = 2;
// As MODE_PLAIN_BMN with fp32 output, stored row by row from the registers
// (the router's gradient products, whose sums stay in fp32).
constexpr int MODE_PLAIN_BMN_F32 = 3;
// The backward of the SwiGLU, fused into the recomputed gate/up pass: the
// accumulator holds g = A W1^T and u = A W3^T as in MODE_SWIGLU_BF16, the
// epilogue reads dH [rows, F] and writes dG = dH u silu'(g) and dU = dH
// silu(g) into C = [dG | dU] [rows, 2F], bf16.
constexpr int MODE_SWIGLU_BWD = 4;

struct GemmArgs {
  const int32_t* offsets;  // [G+1] device, or nullptr: one group [0, rows_single)
  int num_groups;
  int rows_single;
  int n_per_group;         // output columns per group (= B rows per group)
  int K;
  void* C;
  int ldc;                 // elements
  uint32_t* status;
  const int32_t* gather_rows;  // GATHER: A row of output row r is gather_src[gather_rows[r]]
  const void* gather_src;      // GATHER: [rows, K] bf16
  int m_fastest;               // tile order inside a group: 1 = m-tiles fastest
  int kb_split;                // PLAIN_BMN: k-blocks read from B0, the rest from B1
  int b0_rows;                 // PLAIN_BMN: K rows of a group in B0
  int b1_rows;                 // PLAIN_BMN: K rows of a group in B1
  // CTA-pair kernel: one extra group after the routed ones, with tensors of
  // its own (the shared expert over all tokens), or x_rows = 0
  int x_rows;                  // its rows (A rows from 0)
  int x_n;                     // its output columns (B rows per half as above)
  int x_K;                     // its K
  void* x_C;                   // its output
  int x_ldc;
  int gather_limit;            // GATHER: entries of gather_rows
  int gather_src_rows;         // GATHER: rows of gather_src
  const void* aux;             // SWIGLU_BWD: dH [rows, n_per_group] bf16
  // Combine folded into a plain pass (null: not folded).  C is y_perm [R,
  // n], x_C the shared expert's y_sh [T, n] (or no extra group).  For each
  // (token, output tile) fold_cnt counts the rows written; the warp whose
  // row brings it to fold_target (k, plus 1 with a shared expert) forms
  // out[t] = y_sh[t] + sum_j w[t, j] y_perm[slot[t, j]] over those columns,
  // in j order, as the separate combine would.
  int32_t* fold_cnt;           // [T, fold_nt], the token's skipped pairs at launch
  int fold_nt;
  int fold_T;
  int fold_target;
  int fold_k;
  const int32_t* fold_src;     // perm_src [R]: token of each routed row
  const int32_t* fold_slot;    // slot_pos [T, k]
  const float* fold_w;         // topk_w [T, k]
  void* fold_out;              // out [T, n] bf16
  // A rows filled by the launch itself (gate/up, null: A is complete at
  // launch).  Warps 6.. copy row r of A (cp_dst) from row cp_perm[r] of
  // cp_src, in increasing row order over all CTAs, and add the rows to
  // cp_ready[1 + r / 32] once they are stored; a producer waits for the blocks
  // of its tile's A rows before loading them.
  const void* cp_src;          // x [cp_src_rows, K] bf16
  const int32_t* cp_perm;      // perm_src [rows]
  int32_t* cp_ready;           // [1 + ceil(rows / 32)]: next unit, block counts; zero at launch
  void* cp_dst;                // A = x_perm [rows, K] bf16
  int cp_src_rows;
};

// Where a tile of the CTA-pair kernel lies: a routed group's (m, n) tile, or
// one of the extra group's (tiles after all routed ones, n fastest).
struct PairTile {
  bool x;        // the extra group
  int g, m, n;
  int row0;      // first row of the group in its A and C tensors
  int rows;      // rows of the group
  int kblocks;
};

// silu(g) = g / (1 + e^-g) with the fast exponential and the fast divide
// (a reciprocal and a multiply, no IEEE slow path): a few ulp of fp32, far
// below the bf16 rounding of h that follows.  For g < -87, e^-g overflows
// and the quotient is 0, the limit of silu.
__device__ __forceinline__ float silu_f32(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// One warp computes per-group tile prefixes: prefix[g] = sum_{g' < g} m_tiles(g') * n_tiles,
// with m-tiles of TM rows.
template <int TM = BM>
__device__ void build_tile_prefix(const GemmArgs& a, int n_tiles, int* s_off, int* s_prefix) {
  const int lane = threadIdx.x & 31;
  const int G = a.num_groups;
  if (a.offsets == nullptr) {
    if (lane == 0) {
      s_off[0] = 0;
      s_off[1] = a.rows_single;
      s_prefix[0] = 0;
      s_prefix[1] = ((a.rows_single + TM - 1) / TM) * n_tiles;
    }
    __syncwarp();
    return;
  }
  for (int i = lane; i <= G; i += 32) s_off[i] = a.offsets[i];
  __syncwarp();
  const int per = (G + 31) / 32;
  const int g0 = lane * per;
  int local = 0;
  for (int g = g0; g < g0 + per && g < G; ++g) {
    const int rows = s_off[g + 1] - s_off[g];
    local += ((rows > 0 ? rows : 0) + TM - 1) / TM * n_tiles;
  }
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  int run = incl - local;
  for (int g = g0; g < g0 + per && g < G; ++g) {
    s_prefix[g] = run;
    const int rows = s_off[g + 1] - s_off[g];
    run += ((rows > 0 ? rows : 0) + TM - 1) / TM * n_tiles;
  }
  if (lane == 31) s_prefix[G] = incl;
  __syncwarp();
}

// Tile order inside a group.  n fastest (default): the CTAs running at the
// same time share A tiles and one expert's weights, which suits experts whose
// weights fit in L2 many times over.  m fastest: they share B tiles instead,
// so an expert whose weights are a large part of L2 is streamed from HBM
// once while its (smaller) rows are re-read from L2.
template <int TM = BM>
__device__ __forceinline__ void tile_mn(int local, int rows_g, int n_tiles, int m_fastest,
                                        int& m, int& n) {
  if (m_fastest) {
    const int mt = (rows_g + TM - 1) / TM;
    n = local / mt;
    m = local - n * mt;
  } else {
    m = local / n_tiles;
    n = local - m * n_tiles;
  }
}

// Largest g with prefix[g] <= tile (groups with no tiles are skipped).
__device__ __forceinline__ int find_group(const int* s_prefix, int G, int tile) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_prefix[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// --------------------------------------------------- CTA-pair (2-SM) kernel
// The same grouped GEMM with a cluster of two CTAs per 256 x BN_ACC tile:
// rank r holds rows [128 r, 128 r + 128) of the A tile and half of the B tile
// (SwiGLU: rank 0 the W1 rows, rank 1 the W3 rows; plain: rows
// [r BN_ACC/2, (r+1) BN_ACC/2)), so each SM stages half the B bytes of the
// single-CTA kernel per MMA flop.  Rank 0 issues tcgen05.mma.cta_group::2
// (M = 256), which reads both CTAs' shared memory and writes each CTA's 128
// accumulator rows into its own TMEM; commits arrive on both CTAs'
// barriers.  Both CTAs' TMA completions are counted on rank 0's stage
// barrier.  No load uses cluster multicast.
constexpr int BM2 = 256;

// BN_ACC accumulator columns per tile (gate and up columns together for
// SwiGLU).  Up to 256 the TMEM accumulator is double buffered, so the
// epilogue of a tile overlaps the MMAs of the next.  BN_ACC = 512 fills TMEM
// with one accumulator of two N = 256 halves (two MMAs per K step): each
// staged byte of A then feeds twice the MMA work, which matters because the
// tiles are streamed from L2; the producer keeps prefetching the next
// tile's stages while the epilogue drains the accumulator.
template <int BN_ACC>
struct PairCfg {
  static constexpr int NSUB = BN_ACC > 256 ? BN_ACC / 256 : 1;   // MMAs per K step
  static constexpr int N_MMA = BN_ACC / NSUB;                     // N of one MMA
  static constexpr int NACC = BN_ACC > 256 ? 1 : 2;               // TMEM buffers
  static constexpr int B_HALF_BYTES = (BN_ACC / 2) * BK * 2;
  static constexpr int STAGE_BYTES = A_STAGE_BYTES + B_HALF_BYTES;
  static constexpr int STAGES = (196608 / STAGE_BYTES) > 8 ? 8 : (196608 / STAGE_BYTES);
  static constexpr int TMEM_COLS = NACC * BN_ACC;
  static constexpr int EPI_BYTES = 4 * 32 * 128;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_BYTES + 1024 + 1024;
  static_assert(TMEM_COLS <= 512, "TMEM holds 512 columns");
};

template <int BN_OUT>
__device__ __forceinline__ int extra_tiles(const GemmArgs& a) {
  return a.x_rows > 0 ? (a.x_rows + BM2 - 1) / BM2 * ((a.x_n + BN_OUT - 1) / BN_OUT) : 0;
}

// Whether `tile` is one of the extra group's.  They follow the routed
// groups' tiles, except under the folded combine (XFIRST), where they come
// first: every token's output waits for its shared-expert row, so those
// rows are done early.
template <bool XFIRST>
__device__ __forceinline__ bool is_extra_tile(int routed_tiles, int x_tiles, int tile) {
  return XFIRST ? tile < x_tiles : tile >= routed_tiles;
}

template <int BN_OUT, bool XFIRST>
__device__ __forceinline__ PairTile pair_tile(const GemmArgs& a, const int* s_off,
                                              const int* s_prefix, int G, int n_tiles, int tile) {
  PairTile t;
  const int xt = extra_tiles<BN_OUT>(a);
  if (is_extra_tile<XFIRST>(s_prefix[G], xt, tile)) {
    const int local = XFIRST ? tile : tile - s_prefix[G];
    const int xn = (a.x_n + BN_OUT - 1) / BN_OUT;
    t.x = true;
    t.g = 0;
    t.m = local / xn;
    t.n = local - t.m * xn;
    t.row0 = 0;
    t.rows = a.x_rows;
    t.kblocks = a.x_K / BK;
  } else {
    if (XFIRST) tile -= xt;
    t.x = false;
    t.g = find_group(s_prefix, G, tile);
    t.row0 = s_off[t.g];
    t.rows = s_off[t.g + 1] - s_off[t.g];
    tile_mn<BM2>(tile - s_prefix[t.g], t.rows, n_tiles, a.m_fastest, t.m, t.n);
    t.kblocks = a.K / BK;
  }
  return t;
}

// Folded combine, run by an epilogue warp once it has stored its 32 rows of
// an output tile (columns [n BN_OUT, (n+1) BN_OUT) clipped to ncols).  The
// stores are completed and published (TMA stores waited for, then a release
// fence), each row's token takes a count for this column tile, and a warp
// whose row brings a token to fold_target forms that token's output columns:
// out[t] = y_sh[t] + sum_j w[t, j] y_perm[slot[t, j]], fp32 in j order, as
// combine_kernel does, from L2 (the rows were written by other CTAs).  All
// control flow around the shuffles is warp-uniform.
template <int BN_OUT>
__device__ __forceinline__ void fold_combine_rows(const GemmArgs& a, bool extra, int n, int ncols,
                                                  bool valid, int warp_row0, int lane) {
  if (lane == 0) bulk_wait_all();   // this warp's TMA stores have completed
  __syncwarp();
  __threadfence();                  // release: the rows before their counts
  int t = -1;
  if (valid) t = extra ? warp_row0 + lane : __ldg(a.fold_src + warp_row0 + lane);
  bool last = false;
  if (t >= 0 && t < a.fold_T) {
    const int old = atomicAdd(a.fold_cnt + static_cast<size_t>(t) * a.fold_nt + n, 1);
    last = old == a.fold_target - 1;
  }
  uint32_t todo = __ballot_sync(0xffffffffu, last);
  if (todo == 0u) return;
  __threadfence();   // acquire: the other rows of these tokens are visible from here on
  const int k = a.fold_k;
  const __nv_bfloat16* yp = static_cast<const __nv_bfloat16*>(a.C);
  const __nv_bfloat16* ysh = static_cast<const __nv_bfloat16*>(a.x_C);
  __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.fold_out);
  const long long rmax = static_cast<long long>(a.fold_T) * k;
  while (todo != 0u) {
    const int src = __ffs(todo) - 1;
    todo &= todo - 1u;
    const int tt = __shfl_sync(0xffffffffu, t, src);
    int my_slot = -1;
    float my_w = 0.f;
    if (lane < k) {
      my_slot = a.fold_slot[static_cast<size_t>(tt) * k + lane];
      my_w = a.fold_w[static_cast<size_t>(tt) * k + lane];
      if (static_cast<long long>(my_slot) >= rmax) my_slot = -1;
    }
    // lanes whose columns lie past ncols (a partial last tile) load and
    // store nothing but still take part in the shuffles
    for (int c0 = 0; c0 < BN_OUT; c0 += 256) {
      const int col = n * BN_OUT + c0 + lane * 8;
      const bool in = col < ncols;
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.f;
      if (ysh != nullptr && in) {
        const uint4 v =
            __ldcg(reinterpret_cast<const uint4*>(ysh + static_cast<size_t>(tt) * a.x_ldc + col));
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = __bfloat1622float2(h[i]);
          acc[2 * i] = f.x;
          acc[2 * i + 1] = f.y;
        }
      }
      for (int j0 = 0; j0 < k; j0 += 8) {
        uint4 v[8];
        float wj[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int j = j0 + q;
          const int sl = __shfl_sync(0xffffffffu, my_slot, j & 31);
          wj[q] = __shfl_sync(0xffffffffu, my_w, j & 31);
          v[q] = (in && j < k && sl >= 0)
                     ? __ldcg(reinterpret_cast<const uint4*>(yp + static_cast<size_t>(sl) * a.ldc +
                                                             col))
                     : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (j0 + q >= k) break;
          const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v[q]);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(h[i]);
            acc[2 * i] = fmaf(wj[q], f.x, acc[2 * i]);
            acc[2 * i + 1] = fmaf(wj[q], f.y, acc[2 * i + 1]);
          }
        }
      }
      uint4 o;
      uint32_t* op = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
      for (int i = 0; i < 4; ++i) op[i] = pack_bf16x2(acc[2 * i], acc[2 * i + 1]);
      if (in) *reinterpret_cast<uint4*>(out + static_cast<size_t>(tt) * ncols + col) = o;
    }
  }
}

// Copy role of a gate/up launch that fills its own A rows (see GemmArgs).
// The rows go in 8-row units handed out in increasing order by a counter
// (cp_ready[0]), so they complete roughly in the order the
// tiles consume them, and only running warps take work: a producer never
// waits for a CTA that is not resident.  Each warp asks for its next unit
// before copying the current one, hiding the counter's latency.  x rows
// are loaded with an L2 evict-last hint (each is read k times).  After a
// unit's stores every lane fences, and lane 0 (fencing again after the warp
// barrier) adds the rows to their 32-row block's count.
__device__ __forceinline__ void copy_a_rows(const GemmArgs& a, int rows, int lane) {
  const int vecs = a.K / 8;   // 16-byte pieces per row
  const uint4* src = static_cast<const uint4*>(a.cp_src);
  uint4* dst = static_cast<uint4*>(a.cp_dst);
  const uint64_t keep = l2_policy_evict_last();
  const int units = (rows + 7) / 8;
  int* next = a.cp_ready;
  int u = 0;
  if (lane == 0) u = atomicAdd(next, 1);
  u = __shfl_sync(0xffffffffu, u, 0);
  while (u < units) {
    int nu = 0;
    if (lane == 0) nu = atomicAdd(next, 1);
    const int r0 = u * 8;
    const int nr = rows - r0 < 8 ? rows - r0 : 8;
    for (int h = 0; h < 8; h += 4) {
      size_t sb[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int r = r0 + h + q < rows ? r0 + h + q : rows - 1;
        int t = __ldg(a.cp_perm + r);
        t = (t < 0 || t >= a.cp_src_rows) ? 0 : t;
        sb[q] = static_cast<size_t>(t) * vecs;
      }
      for (int c0 = 0; c0 < vecs; c0 += 128) {
        uint4 v[4][4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int c = c0 + lane + 32 * j;
            v[q][j] =
                c < vecs ? ld_global_hint(src + sb[q] + c, keep) : make_uint4(0u, 0u, 0u, 0u);
          }
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int c = c0 + lane + 32 * j;
            if (c < vecs && h + q < nr) dst[static_cast<size_t>(r0 + h + q) * vecs + c] = v[q][j];
          }
      }
    }
    __threadfence();
    __syncwarp();
    if (lane == 0) {
      __threadfence();
      atomicAdd(a.cp_ready + 1 + r0 / 32, nr);
    }
    u = __shfl_sync(0xffffffffu, nu, 0);
  }
}

// Producer side: wait (bounded) until the A rows [lo, hi) of a tile are
// stored, then order the later TMA loads after that observation.  `rows`
// is the copied total (blocks before the last hold 32 rows).
__device__ __forceinline__ bool wait_a_rows(const GemmArgs& a, int lo, int hi, int rows,
                                            volatile int* abort_flag) {
  if (lo >= hi) return true;
  const unsigned long long t0 = globaltimer_ns();
  for (int b = lo / 32; b <= (hi - 1) / 32; ++b) {
    const int need = rows - 32 * b < 32 ? rows - 32 * b : 32;
    while (ld_acquire_gpu(a.cp_ready + 1 + b) < need) {
      if (*abort_flag) return false;
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        *abort_flag = 1;
        return false;
      }
    }
  }
  fence_proxy_async_global();
  return true;
}

// L2 hints of the pair kernel: the output tiles (h, y_perm: not read again
// by this kernel) are stored evict-first so they do not push out the A and
// B tiles that the other n-tile / m-tile pairs are about to re-read; A tiles
// can be loaded evict-last.
constexpr bool kStoreEvictFirst = true;
constexpr bool kLoadAEvictLast = false;

template <int BN_ACC, int MODE, int VAR>
__global__ void __cluster_dims__(2, 1, 1)
__launch_bounds__(VAR == VAR_COPY ? NUM_THREADS_COPY : NUM_THREADS, 1)
grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                         const __grid_constant__ CUtensorMap tmB0,
                         const __grid_constant__ CUtensorMap tmB1,
                         const __grid_constant__ CUtensorMap tmC,
                         const __grid_constant__ CUtensorMap tmA2,
                         const __grid_constant__ CUtensorMap tmB0_2,
                         const __grid_constant__ CUtensorMap tmB1_2,
                         const __grid_constant__ CUtensorMap tmC2, const GemmArgs args) {
  using Cfg = PairCfg<BN_ACC>;
  constexpr int STAGES = Cfg::STAGES;
  constexpr bool GATHER = VAR == VAR_GATHER;
  constexpr bool COPY = VAR == VAR_COPY;
  constexpr bool FOLD = VAR == VAR_FOLD;
  static_assert(!(GATHER || COPY) || MODE == MODE_SWIGLU_BF16, "gate/up variants");
  static_assert(!FOLD || MODE == MODE_PLAIN_BF16, "plain-mode variant");
  constexpr bool SWI_BWD = MODE == MODE_SWIGLU_BWD;
  constexpr bool SWIGLU = MODE == MODE_SWIGLU_BF16 || SWI_BWD;
  constexpr bool BMN = MODE == MODE_PLAIN_BMN || MODE == MODE_PLAIN_BMN_F32;
  constexpr bool OUT_F32 = MODE == MODE_PLAIN_BMN_F32;
  constexpr int BN_OUT = SWIGLU ? BN_ACC / 2 : BN_ACC;
  constexpr int NSUB = Cfg::NSUB;
  constexpr int NACC = Cfg::NACC;
  constexpr uint32_t IDESC = idesc_bf16_f32(BM2, Cfg::N_MMA, BMN);
  constexpr int BOX_MN = 64 * 128;   // PLAIN_BMN: one 64-column box of 64 k-rows


  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* smemA = smem;
  uint8_t* smemB = smem + STAGES * A_STAGE_BYTES;
  uint8_t* smemEpi = smem + STAGES * Cfg::STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smemEpi + Cfg::EPI_BYTES);
  uint64_t* full_bar = bars;                   // rank 0's copy is used
  uint64_t* empty_bar = bars + STAGES;         // both copies
  uint64_t* tfull_bar = bars + 2 * STAGES;     // both copies
  uint64_t* tempty_bar = bars + 2 * STAGES + 2;  // rank 0's copy (8 arrivals)
  uint64_t* drain_bar = bars + 2 * STAGES + 4;

  __shared__ int s_off[MAX_GROUPS + 1];
  __shared__ int s_prefix[MAX_GROUPS + 1];
  __shared__ uint32_t s_tmem_base;
  __shared__ int s_abort;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;
  const int n_tiles = (args.n_per_group + BN_OUT - 1) / BN_OUT;   // a last tile may be partial
  const int G = args.offsets == nullptr ? 1 : args.num_groups;

  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull_bar[a], 1);
      mbar_init(&tempty_bar[a], 8);
    }
    mbar_init(drain_bar, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB0);
    if (SWIGLU || BMN) tma_prefetch_desc(&tmB1);
    tma_prefetch_desc(&tmC);
    if (args.x_rows > 0) {
      tma_prefetch_desc(&tmA2);
      tma_prefetch_desc(&tmB0_2);
      if (SWIGLU) tma_prefetch_desc(&tmB1_2);
      tma_prefetch_desc(&tmC2);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(&s_tmem_base, Cfg::TMEM_COLS);
    tmem_relinquish_pair();
  }
  pdl_wait();   // everything above touches no global memory
  if (warp == 2) build_tile_prefix<BM2>(args, n_tiles, s_off, s_prefix);
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();        // both CTAs' barriers are initialised
  tc_fence_after();

  const uint32_t tmem_base = s_tmem_base;
  const int x_tiles = extra_tiles<BN_OUT>(args);
  const int total_tiles = s_prefix[G] + x_tiles;
  volatile int* abort_flag = &s_abort;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // Lane 0 waits for free stages, arms the barrier and loads B (and A
    // tiles).  GATHER: the A rows of a routed tile are gathered from x by
    // the permutation instead, every lane fetching four rows per stage with
    // one tile::gather4 load (row r of the tile, r = 4 lane + q, is token
    // gather_rows[first row + r], clamped into range; rows past the group
    // load a valid row whose result is never stored).
    int stage = 0;
    uint32_t phase = 0, issued_mask = 0, issued_phase = 0;
    bool ok = true;
    const uint64_t a_policy = kLoadAEvictLast ? l2_policy_evict_last() : 0ull;
    // without gathers lane 0 alone drives the ring
    for (int tile = pair; tile < total_tiles && ok && (GATHER || lane == 0); tile += npairs) {
      const PairTile pt = pair_tile<BN_OUT, FOLD>(args, s_off, s_prefix, G, n_tiles, tile);
      const int g = pt.g, n = pt.n, kblocks = pt.kblocks;
      const int arow = pt.row0 + pt.m * BM2 + static_cast<int>(rank) * BM;
      const int gbase = pt.x ? 0 : g * args.n_per_group;
      const int brow = SWIGLU ? gbase + n * BN_OUT
                              : gbase + n * BN_OUT + static_cast<int>(rank) * (BN_ACC / 2);
      const CUtensorMap* ma = pt.x ? &tmA2 : &tmA;
      const CUtensorMap* mb = (SWIGLU && rank == 1) ? (pt.x ? &tmB1_2 : &tmB1)
                                                    : (pt.x ? &tmB0_2 : &tmB0);
      const bool gathered = GATHER && !pt.x;
      if constexpr (COPY) {
        // lane 0 alone runs this loop here
        if (!pt.x &&
            !wait_a_rows(args, arow, min(arow + BM, pt.row0 + pt.rows), s_off[G], abort_flag)) {
          ok = false;
          break;
        }
      }
      int tok[4] = {0, 0, 0, 0};
      if (gathered) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          int r = arow + 4 * lane + q;
          r = r < args.gather_limit ? r : args.gather_limit - 1;
          const int t = __ldg(args.gather_rows + r);
          tok[q] = t < 0 ? 0 : (t >= args.gather_src_rows ? args.gather_src_rows - 1 : t);
        }
      }
      for (int kb = 0; kb < kblocks; ++kb) {
        bool w_ok = true;
        if (lane == 0) w_ok = mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag);
        if (GATHER) w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
        if (!w_ok) { ok = false; break; }
        if (lane == 0) {
          if (rank == 0) mbar_arrive_expect_tx(&full_bar[stage], 2 * Cfg::STAGE_BYTES);
          if (!gathered) {
            if (kLoadAEvictLast)
              tma_load_2d_pair_hint(smemA + stage * A_STAGE_BYTES, ma, &full_bar[stage], kb * BK,
                                    arow, a_policy);
            else
              tma_load_2d_pair(smemA + stage * A_STAGE_BYTES, ma, &full_bar[stage], kb * BK,
                               arow);
          }
          if (BMN) {
            // this CTA's BN_ACC/2 columns of B, 64 columns (one box) at a time
            const bool first = kb < args.kb_split;
            const CUtensorMap* mbk = first ? &tmB0 : &tmB1;
            const int krow = first ? g * args.b0_rows + kb * BK
                                   : g * args.b1_rows + (kb - args.kb_split) * BK;
            const int col0 = n * BN_ACC + static_cast<int>(rank) * (BN_ACC / 2);
#pragma unroll
            for (int j = 0; j < BN_ACC / 128; ++j)
              tma_load_2d_pair(smemB + stage * Cfg::B_HALF_BYTES + j * BOX_MN, mbk,
                               &full_bar[stage], col0 + j * 64, krow);
          } else {
            tma_load_2d_pair(smemB + stage * Cfg::B_HALF_BYTES, mb, &full_bar[stage], kb * BK,
                             brow);
          }
        }
        if (gathered)
          tma_gather4_pair(smemA + stage * A_STAGE_BYTES + lane * 512, ma, &full_bar[stage],
                           kb * BK, tok[0], tok[1], tok[2], tok[3]);
        issued_mask |= 1u << stage;
        issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
    }
    if (lane == 0) {
      pdl_trigger();   // all loads issued: the next kernel may launch
      if (!ok && rank == 0) {
        // rank 0's stage barriers count both CTAs' copies: let them all land
        for (int s = 0; s < STAGES; ++s) {
          if (!(issued_mask & (1u << s))) continue;
          const uint32_t par = (issued_phase >> s) & 1u;
          const unsigned long long t0 = globaltimer_ns();
          while (!mbar_try_wait(&full_bar[s], par))
            if (globaltimer_ns() - t0 > kWaitLimitNs) break;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------- MMA issuer (rank 0)
    if (lane == 0 && rank == 0) {
      int stage = 0, it = 0;
      uint32_t phase = 0;
      bool ok = true, issued_any = false;
      for (int tile = pair; tile < total_tiles && ok; tile += npairs, ++it) {
        const int acc = it % NACC;
        const uint32_t acc_phase = (it / NACC) & 1;
        const int kblocks =
            is_extra_tile<FOLD>(s_prefix[G], x_tiles, tile) ? args.x_K / BK : args.K / BK;
        if (!mbar_wait(&tempty_bar[acc], acc_phase ^ 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN_ACC;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smemA + stage * A_STAGE_BYTES);
          const uint32_t b_addr = smem_u32(smemB + stage * Cfg::B_HALF_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
#pragma unroll
            for (int sub = 0; sub < NSUB; ++sub) {  // sub-tile: B rows [128 sub, 128 sub + 128)
              const uint32_t bsub = b_addr + sub * (Cfg::N_MMA / 2) * 128;
              const uint64_t bd = BMN ? smem_desc_sw128_mn(bsub + kk * 16 * 128, BOX_MN)
                                      : smem_desc_sw128(bsub + kk * 32);
              tc_mma_f16_pair(d_tmem + sub * Cfg::N_MMA, smem_desc_sw128(a_addr + kk * 32), bd,
                              IDESC, (kb | kk) != 0 ? 1u : 0u);
            }
          issued_any = true;
          tc_commit_pair(&empty_bar[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit_pair(&tfull_bar[acc]);
      }
      if (!ok && issued_any) {
        tc_commit_pair(drain_bar);
        const unsigned long long t0 = globaltimer_ns();
        while (!mbar_try_wait(drain_bar, 0))
          if (globaltimer_ns() - t0 > kWaitLimitNs) break;
      }
    }
  } else if (!COPY || warp < NUM_THREADS / 32) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const uint64_t c_policy = kStoreEvictFirst ? l2_policy_evict_first() : 0ull;
    int it = 0;
    for (int tile = pair; tile < total_tiles; tile += npairs, ++it) {
      const int acc = it % NACC;
      const uint32_t acc_phase = (it / NACC) & 1;
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&tfull_bar[acc], acc_phase, abort_flag));
      if (!ok) break;
      tc_fence_after();
      const PairTile pt = pair_tile<BN_OUT, FOLD>(args, s_off, s_prefix, G, n_tiles, tile);
      const int rows_g = pt.rows, n = pt.n;
      const int r0 = pt.m * BM2 + static_cast<int>(rank) * BM;   // first row (in group) of this CTA
      const bool valid = (r0 + q * 32 + lane) < rows_g;
      const bool warp_full = (r0 + q * 32 + 32) <= rows_g;
      const int warp_row0 = pt.row0 + r0 + q * 32;
      uint8_t* stage_buf = smemEpi + (warp - 2) * (32 * 128);
      const CUtensorMap* mc = pt.x ? &tmC2 : &tmC;
      __nv_bfloat16* cbase = static_cast<__nv_bfloat16*>(pt.x ? args.x_C : args.C);
      const size_t crow_off =
          static_cast<size_t>(warp_row0 + lane) * (pt.x ? args.x_ldc : args.ldc);
      const uint32_t t_addr = tmem_base + acc * BN_ACC + (static_cast<uint32_t>(q * 32) << 16);
      constexpr int UP = Cfg::N_MMA / 2;   // up columns follow the gate columns
      // output columns of the group: a last partial n-tile (plain mode, the
      // columns a multiple of 64) skips its 64-column chunks past them
      const int ncols = pt.x ? args.x_n : args.n_per_group;
#pragma unroll 1
      for (int cb = 0; cb < BN_OUT / 64; ++cb) {
        // accumulator column of this 64-column chunk and its output column:
        // sub-tile `sub` holds N_MMA columns, its first half from rank 0's B
        // rows and its second half from rank 1's (SwiGLU: gate, then up)
        int acol, ocol;
        if (SWIGLU) {
          const int sub = (cb * 64) / (Cfg::N_MMA / 2);
          const int c = (cb * 64) % (Cfg::N_MMA / 2);
          acol = sub * Cfg::N_MMA + c;
          ocol = n * BN_OUT + cb * 64;
        } else {
          const int sub = (cb * 64) / Cfg::N_MMA;
          const int jj = (cb * 64) % Cfg::N_MMA;
          acol = cb * 64;
          ocol = n * BN_ACC + (jj / (Cfg::N_MMA / 2)) * (BN_ACC / 2) + sub * (Cfg::N_MMA / 2) +
                 jj % (Cfg::N_MMA / 2);
        }
        if (ocol >= ncols) continue;   // warp-uniform
        uint32_t packed[32];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int c0 = acol + half * 32;
          uint32_t v[32];
          if (SWIGLU) {
            uint32_t u[32];
            tmem_ld16(t_addr + c0, *reinterpret_cast<uint32_t(*)[16]>(&v[0]));
            tmem_ld16(t_addr + c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&v[16]));
            tmem_ld16(t_addr + UP + c0, *reinterpret_cast<uint32_t(*)[16]>(&u[0]));
            tmem_ld16(t_addr + UP + c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&u[16]));
            tmem_ld_wait();
            if constexpr (SWI_BWD) {
              if (valid) {
                // dH of these 32 columns of the row; dG and dU as the
                // SwiGLU backward: s = sigmoid(g), dU = dH g s,
                // dG = dH u s (1 + g (1 - s))
                const size_t rr = static_cast<size_t>(warp_row0 + lane);
                const uint4* dhp = reinterpret_cast<const uint4*>(
                    static_cast<const __nv_bfloat16*>(args.aux) + rr * args.n_per_group + ocol +
                    half * 32);
                uint4 dq[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) dq[i] = dhp[i];
                const __nv_bfloat162* dh2 = reinterpret_cast<const __nv_bfloat162*>(dq);
                uint32_t pg[16], pu[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                  const float2 dh = __bfloat1622float2(dh2[i]);
                  float dgv[2], duv[2];
#pragma unroll
                  for (int e = 0; e < 2; ++e) {
                    const float g = __uint_as_float(v[2 * i + e]);
                    const float uu = __uint_as_float(u[2 * i + e]);
                    const float sg = __fdividef(1.0f, 1.0f + __expf(-g));
                    const float d = e ? dh.y : dh.x;
                    duv[e] = d * g * sg;
                    dgv[e] = d * uu * (sg * (1.0f + g * (1.0f - sg)));
                  }
                  pg[i] = pack_bf16x2(dgv[0], dgv[1]);
                  pu[i] = pack_bf16x2(duv[0], duv[1]);
                }
                uint4* dg_dst = reinterpret_cast<uint4*>(cbase + crow_off + ocol + half * 32);
                uint4* du_dst = reinterpret_cast<uint4*>(cbase + crow_off + args.n_per_group +
                                                         ocol + half * 32);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  dg_dst[i] = make_uint4(pg[4 * i], pg[4 * i + 1], pg[4 * i + 2], pg[4 * i + 3]);
                  du_dst[i] = make_uint4(pu[4 * i], pu[4 * i + 1], pu[4 * i + 2], pu[4 * i + 3]);
                }
              }
              continue;
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float h0 = silu_f32(__uint_as_float(v[2 * i])) * __uint_as_float(u[2 * i]);
              const float h1 =
                  silu_f32(__uint_as_float(v[2 * i + 1])) * __uint_as_float(u[2 * i + 1]);
              packed[half * 16 + i] = pack_bf16x2(h0, h1);
            }
          } else {
            tmem_ld16(t_addr + c0, *reinterpret_cast<uint32_t(*)[16]>(&v[0]));
            tmem_ld16(t_addr + c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&v[16]));
            tmem_ld_wait();
            if constexpr (OUT_F32) {
              if (valid) {
                float4* dst = reinterpret_cast<float4*>(
                    static_cast<float*>(pt.x ? args.x_C : args.C) + crow_off + ocol + half * 32);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                  dst[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                       __uint_as_float(v[4 * i + 2]),
                                       __uint_as_float(v[4 * i + 3]));
              }
            } else {
#pragma unroll
              for (int i = 0; i < 16; ++i)
                packed[half * 16 + i] =
                    pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
            }
          }
        }
        if constexpr (OUT_F32 || SWI_BWD) continue;   // stored above
        if (warp_full) {
          if (lane == 0) bulk_wait_read_all();
          __syncwarp();
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(stage_buf + lane * 128 + ((c ^ (lane & 7)) << 4)) =
                make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2],
                           packed[4 * c + 3]);
          fence_async_shared();
          __syncwarp();
          if (lane == 0) {
            if (kStoreEvictFirst)
              tma_store_2d_hint(mc, stage_buf, ocol, warp_row0, c_policy);
            else
              tma_store_2d(mc, stage_buf, ocol, warp_row0);
            bulk_commit();
          }
        } else if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(cbase + crow_off + ocol);
#pragma unroll
          for (int c = 0; c < 8; ++c)
            dst[c] = make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2],
                                packed[4 * c + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_rank0(&tempty_bar[acc]);
      if constexpr (FOLD) fold_combine_rows<BN_OUT>(args, pt.x, n, ncols, valid, warp_row0, lane);
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  } else {
    // ------------------------------------------------- A-row copy (gate/up)
    if constexpr (COPY) copy_a_rows(args, s_off[G], lane);
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();        // neither CTA leaves while the other still uses the pair
  if (threadIdx.x == 0 && s_abort) atomicOr(args.status, kDevTimeout);
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
  }
}

// ----------------------------------------------------------------- host side
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// Looked up once per process; the initialisation of a function-local
// static is thread-safe.
EncodeTiledFn get_encode_fn() {
  static const EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(p);
    return nullptr;
  }();
  return fn;
}

// Row-major bf16 matrix [rows, cols] read in boxes of box_rows x 64 with the
// 128-byte swizzle; rows past `rows` read as zero.
bool make_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(BK), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

int num_sms() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

template <int BN_ACC, int MODE, int VAR = VAR_NONE>
cudaError_t launch_pair(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                        const CUtensorMap& c, const CUtensorMap& a2, const CUtensorMap& b0_2,
                        const CUtensorMap& b1_2, const CUtensorMap& c2, const GemmArgs& args,
                        int rows_upper, cudaStream_t stream, int threads = NUM_THREADS) {
  using Cfg = PairCfg<BN_ACC>;
  constexpr int BN_OUT = MODE == MODE_SWIGLU_BF16 ? BN_ACC / 2 : BN_ACC;
  auto kern = grouped_gemm_pair_kernel<BN_ACC, MODE, VAR>;
  static std::atomic<unsigned long long> attr_done{0};
  int dev = 0;
  cudaGetDevice(&dev);
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(attr_done.load(std::memory_order_acquire) & bit)) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Cfg::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_done.fetch_or(bit, std::memory_order_acq_rel);
  }
  const int G = args.offsets == nullptr ? 1 : args.num_groups;
  GemmArgs a2r = args;
  const double b_bytes = static_cast<double>(BN_OUT == BN_ACC ? args.n_per_group
                                                              : 2 * args.n_per_group) *
                         args.K * 2.0;
  a2r.m_fastest = b_bytes > 32.0 * 1024 * 1024 ? 1 : 0;
  const long long m_tiles_upper = (rows_upper + BM2 - 1) / BM2 + (G > 1 ? G : 0);
  long long tiles_upper = m_tiles_upper * ((args.n_per_group + BN_OUT - 1) / BN_OUT);
  if (args.x_rows > 0)
    tiles_upper += static_cast<long long>((args.x_rows + BM2 - 1) / BM2) *
                   ((args.x_n + BN_OUT - 1) / BN_OUT);
  if (tiles_upper <= 0) return cudaSuccess;
  const int max_pairs = num_sms() / 2;
  const int pairs = static_cast<int>(tiles_upper < max_pairs ? tiles_upper : max_pairs);
  return launch_pdl(kern, dim3(2 * pairs), dim3(threads), Cfg::SMEM_BYTES, stream, a, b0, b1,
                    c, a2, b0_2, b1_2, c2, a2r);
}

}  // namespace

// h[r] = silu(A[r] W1[g]^T) * (A[r] W3[g]^T), bf16 out.  extra: one more
// group with tensors of its own (the shared expert), in the same launch.
cudaError_t grouped_swiglu_gateup_bf16(const void* A, int64_t a_rows, const int32_t* offsets,
                                       int num_groups, int rows_single, const void* W1,
                                       const void* W3, int F, int K, void* H, uint32_t* status,
                                       cudaStream_t stream, const GemmExtraGroup* extra,
                                       const GemmCopy* copy) {
  CUtensorMap ta, tb0, tb1, tc, xa, xb0, xb1, xc;
  const int64_t b_rows = static_cast<int64_t>(offsets ? num_groups : 1) * F;
  const int64_t c_rows = offsets ? a_rows : rows_single;
  // 128 output columns (gate + up = 256 accumulator columns, double
  // buffered) per tile.  Measured on B200: 256 output columns per tile with
  // one 512-column accumulator was slower on every workload (qwen3_30b
  // gate/up 0.92 vs 0.66-0.70 ms): the epilogue is no longer hidden.
  const int bh = 128;   // B rows each CTA of the pair loads
  if (!make_map(&ta, A, a_rows, K, BM) || !make_map(&tb0, W1, b_rows, K, bh) ||
      !make_map(&tb1, W3, b_rows, K, bh) || !make_map(&tc, H, c_rows, F, 32))
    return cudaErrorInvalidValue;
  GemmArgs args{offsets, num_groups, rows_single, F, K, H, F, status, nullptr, nullptr, 0, 0, 0, 0,
                0, 0, 0, nullptr, 0, 0, 0, nullptr};
  if (extra != nullptr && extra->rows > 0) {
    if (!make_map(&xa, extra->A, extra->rows, extra->K, BM) ||
        !make_map(&xb0, extra->B0, extra->n, extra->K, bh) ||
        !make_map(&xb1, extra->B1, extra->n, extra->K, bh) ||
        !make_map(&xc, extra->C, extra->rows, extra->n, 32))
      return cudaErrorInvalidValue;
    args.x_rows = extra->rows;
    args.x_n = extra->n;
    args.x_K = extra->K;
    args.x_C = extra->C;
    args.x_ldc = extra->n;
  } else {
    xa = ta; xb0 = tb0; xb1 = tb1; xc = tc;
  }
  if (copy != nullptr) {
    if (offsets == nullptr || !copy->src || !copy->perm || !copy->ready || copy->src_rows < 1 ||
        (reinterpret_cast<uintptr_t>(copy->src) & 15) || (reinterpret_cast<uintptr_t>(A) & 15))
      return cudaErrorInvalidValue;
    args.cp_src = copy->src;
    args.cp_perm = copy->perm;
    args.cp_ready = copy->ready;
    args.cp_dst = const_cast<void*>(A);
    args.cp_src_rows = copy->src_rows;
  }
  const int rows_upper = offsets ? static_cast<int>(a_rows) : rows_single;
  if (copy != nullptr)
    return launch_pair<256, MODE_SWIGLU_BF16, VAR_COPY>(ta, tb0, tb1, tc, xa, xb0, xb1, xc, args,
                                                        rows_upper, stream, NUM_THREADS_COPY);
  return launch_pair<256, MODE_SWIGLU_BF16>(ta, tb0, tb1, tc, xa, xb0, xb1, xc, args,
                                            rows_upper, stream);
}

// The SwiGLU backward fused into the recomputed gate/up pass: with g and u
// the rows of A W1^T and A W3^T, dGU [rows, 2F] = [dH u silu'(g) | dH silu(g)]
// for dH [rows, F].  Groups as for grouped_swiglu_gateup_bf16.
cudaError_t grouped_swiglu_bwd_bf16(const void* A, int64_t a_rows, const int32_t* offsets,
                                    int num_groups, int rows_single, const void* W1,
                                    const void* W3, int F, int K, const void* dH, void* dGU,
                                    uint32_t* status, cudaStream_t stream) {
  if (F % 128) return cudaErrorInvalidValue;
  CUtensorMap ta, tb0, tb1;
  const int64_t b_rows = static_cast<int64_t>(offsets ? num_groups : 1) * F;
  if (!make_map(&ta, A, a_rows, K, BM) || !make_map(&tb0, W1, b_rows, K, 128) ||
      !make_map(&tb1, W3, b_rows, K, 128))
    return cudaErrorInvalidValue;
  GemmArgs args{offsets, num_groups, rows_single, F, K, dGU, 2 * F, status, nullptr, nullptr, 0,
                0, 0, 0, 0, 0, 0, nullptr, 0, 0, 0, dH};
  const int rows_upper = offsets ? static_cast<int>(a_rows) : rows_single;
  return launch_pair<256, MODE_SWIGLU_BWD>(ta, tb0, tb1, ta, ta, tb0, tb1, ta, args, rows_upper,
                                           stream);
}

// Gate/up pass whose A rows are gathered from X [x_rows, K]: output row r
// (expert-contiguous order, r < R) reads X[rows[r]] (tile::gather4 loads in
// the CTA-pair kernel).  H is [R, F].  extra as for the plain gate/up pass
// (its A rows are read directly).
cudaError_t grouped_swiglu_gateup_gather_bf16(const void* X, int64_t x_rows, const int32_t* rows,
                                              int64_t R, const int32_t* offsets, int num_groups,
                                              const void* W1, const void* W3, int F, int K,
                                              void* H, uint32_t* status, cudaStream_t stream,
                                              const GemmExtraGroup* extra) {
  CUtensorMap ta, tb0, tb1, tc, xa, xb0, xb1, xc;
  const int64_t b_rows = static_cast<int64_t>(num_groups) * F;
  if (!make_map(&ta, X, x_rows, K, 1) || !make_map(&tb0, W1, b_rows, K, 128) ||
      !make_map(&tb1, W3, b_rows, K, 128) || !make_map(&tc, H, R, F, 32))
    return cudaErrorInvalidValue;
  GemmArgs args{offsets, num_groups, 0, F, K, H, F, status, rows, X, 0, 0, 0, 0,
                0, 0, 0, nullptr, 0, static_cast<int>(R), static_cast<int>(x_rows), nullptr};
  if (extra != nullptr && extra->rows > 0) {
    if (!make_map(&xa, extra->A, extra->rows, extra->K, BM) ||
        !make_map(&xb0, extra->B0, extra->n, extra->K, 128) ||
        !make_map(&xb1, extra->B1, extra->n, extra->K, 128) ||
        !make_map(&xc, extra->C, extra->rows, extra->n, 32))
      return cudaErrorInvalidValue;
    args.x_rows = extra->rows;
    args.x_n = extra->n;
    args.x_K = extra->K;
    args.x_C = extra->C;
    args.x_ldc = extra->n;
  } else {
    xa = ta; xb0 = tb0; xb1 = tb1; xc = tc;
  }
  return launch_pair<256, MODE_SWIGLU_BF16, VAR_GATHER>(ta, tb0, tb1, tc, xa, xb0, xb1, xc,
                                                  args, static_cast<int>(R), stream);
}

// Y[r] = A[r] W2[g]^T, bf16 out; N = output columns per group.  extra: one
// more group (the shared expert's down projection, same N), same launch.
// Output columns per tile of grouped_down_bf16 for N x K: 512 accumulator
// columns (one TMEM buffer) only for long K, where the exposed epilogue is a
// small part of a tile: measured on B200, wide's down GEMM (K = 4352) 0.616
// -> 0.551 ms, but qwen3_30b's (K = 768) 0.33 -> 0.38 ms.  N a multiple of
// 128 but not of 256 (page-2 shape, d = 640): 256-column tiles with a
// half-empty last one beat 128-column tiles, whose A tile is streamed twice
// as often per MMA flop.
int down_tile_cols(int N, int K) {
  return (N % 512 == 0 && K >= 4096) ? 512
         : (N % 256 == 0 || (N % 128 == 0 && N > 256)) ? 256 : 128;
}

cudaError_t grouped_down_bf16(const void* A, int64_t a_rows, const int32_t* offsets,
                              int num_groups, int rows_single, const void* W2, int N, int K,
                              void* Y, uint32_t* status, cudaStream_t stream,
                              const GemmExtraGroup* extra, const GemmFold* fold) {
  CUtensorMap ta, tb, tc, xa, xb, xc;
  const int64_t b_rows = static_cast<int64_t>(offsets ? num_groups : 1) * N;
  const int64_t c_rows = offsets ? a_rows : rows_single;
  const int bn = down_tile_cols(N, K);
  // each CTA of the pair loads half of the B tile
  if (!make_map(&ta, A, a_rows, K, BM) || !make_map(&tb, W2, b_rows, K, bn / 2) ||
      !make_map(&tc, Y, c_rows, N, 32))
    return cudaErrorInvalidValue;
  GemmArgs args{offsets, num_groups, rows_single, N, K, Y, N, status, nullptr, nullptr, 0, 0, 0, 0,
                0, 0, 0, nullptr, 0, 0, 0, nullptr};
  if (extra != nullptr && extra->rows > 0) {
    if (extra->n != N || !make_map(&xa, extra->A, extra->rows, extra->K, BM) ||
        !make_map(&xb, extra->B0, N, extra->K, bn / 2) ||
        !make_map(&xc, extra->C, extra->rows, N, 32))
      return cudaErrorInvalidValue;
    args.x_rows = extra->rows;
    args.x_n = N;
    args.x_K = extra->K;
    args.x_C = extra->C;
    args.x_ldc = N;
  } else {
    xa = ta; xb = tb; xc = tc;
  }
  if (fold != nullptr) {
    const bool shared = extra != nullptr && extra->rows > 0;
    if (fold->nt != (N + bn - 1) / bn || (shared && extra->rows != fold->T) || fold->k < 1 ||
        fold->k > 32 || !fold->cnt || !fold->src || !fold->slot || !fold->w || !fold->out)
      return cudaErrorInvalidValue;
    args.fold_cnt = fold->cnt;
    args.fold_nt = fold->nt;
    args.fold_T = fold->T;
    args.fold_target = fold->k + (shared ? 1 : 0);
    args.fold_k = fold->k;
    args.fold_src = fold->src;
    args.fold_slot = fold->slot;
    args.fold_w = fold->w;
    args.fold_out = fold->out;
  }
  const int rows_upper = offsets ? static_cast<int>(a_rows) : rows_single;
  if (fold != nullptr) {
    if (bn == 512)
      return launch_pair<512, MODE_PLAIN_BF16, VAR_FOLD>(ta, tb, tb, tc, xa, xb, xb, xc, args,
                                                         rows_upper, stream);
    if (bn == 256)
      return launch_pair<256, MODE_PLAIN_BF16, VAR_FOLD>(ta, tb, tb, tc, xa, xb, xb, xc, args,
                                                         rows_upper, stream);
    return launch_pair<128, MODE_PLAIN_BF16, VAR_FOLD>(ta, tb, tb, tc, xa, xb, xb, xc, args,
                                                       rows_upper, stream);
  }
  if (bn == 512)
    return launch_pair<512, MODE_PLAIN_BF16>(ta, tb, tb, tc, xa, xb, xb, xc, args,
                                             rows_upper, stream);
  if (bn == 256)
    return launch_pair<256, MODE_PLAIN_BF16>(ta, tb, tb, tc, xa, xb, xb, xc, args,
                                             rows_upper, stream);
  return launch_pair<128, MODE_PLAIN_BF16>(ta, tb, tb, tc, xa, xb, xb, xc, args,
                                           rows_upper, stream);
}

// Y [rows, N] fp32 = A B_g over the groups of A's rows, B_g the rows
// [g b0_rows, g b0_rows + K) of B0 [b0_total_rows, N] (MN-major; rows past
// b0_total_rows read as zero).  K = b0_rows, a multiple of 64; N a multiple
// of 128.
cudaError_t grouped_gemm_bmn_f32out(const void* A, int64_t a_rows, const int32_t* offsets,
                                    int num_groups, int rows_single, const void* B0,
                                    int b0_rows, int64_t b0_total_rows, int N, float* Y,
                                    uint32_t* status, cudaStream_t stream) {
  const int K = b0_rows;
  if (K % BK || K <= 0 || N % 128 || b0_total_rows <= 0) return cudaErrorInvalidValue;
  CUtensorMap ta, tb0;
  if (!make_map(&ta, A, a_rows, K, BM) || !make_map(&tb0, B0, b0_total_rows, N, BK))
    return cudaErrorInvalidValue;
  GemmArgs args{offsets, num_groups, rows_single, N, K, Y, N, status, nullptr, nullptr, 0,
                K / BK, K, 0, 0, 0, 0, nullptr, 0, 0, 0, nullptr};
  const int rows_upper = offsets ? static_cast<int>(a_rows) : rows_single;
  if (N % 256 == 0)
    return launch_pair<256, MODE_PLAIN_BMN_F32>(ta, tb0, tb0, ta, ta, tb0, tb0, ta, args,
                                                rows_upper, stream);
  return launch_pair<128, MODE_PLAIN_BMN_F32>(ta, tb0, tb0, ta, ta, tb0, tb0, ta, args,
                                              rows_upper, stream);
}

// Y[r] = A[r] B_g with B_g stored [K, N] (MN-major): its first b0_rows rows
// from B0 [G * b0_rows, N], the remaining K - b0_rows from B1 [G * (K -
// b0_rows), N] (B1 may be null when b0_rows == K).  b0_rows a multiple of 64.
cudaError_t grouped_gemm_bmn_bf16(const void* A, int64_t a_rows, const int32_t* offsets,
                                  int num_groups, int rows_single, const void* B0,
                                  const void* B1, int b0_rows, int N, int K, void* Y,
                                  uint32_t* status, cudaStream_t stream) {
  if (b0_rows % BK || b0_rows > K || (b0_rows < K && B1 == nullptr) || N % 128)
    return cudaErrorInvalidValue;
  CUtensorMap ta, tb0, tb1, tc;
  const int64_t G = offsets ? num_groups : 1;
  const int64_t c_rows = offsets ? a_rows : rows_single;
  const int b1_rows = K - b0_rows;
  if (!make_map(&ta, A, a_rows, K, BM) || !make_map(&tb0, B0, G * b0_rows, N, BK) ||
      !make_map(&tb1, b1_rows ? B1 : B0, G * (b1_rows ? b1_rows : b0_rows), N, BK) ||
      !make_map(&tc, Y, c_rows, N, 32))
    return cudaErrorInvalidValue;
  GemmArgs args{offsets, num_groups, rows_single, N, K, Y, N, status, nullptr, nullptr, 0,
                b0_rows / BK, b0_rows, b1_rows, 0, 0, 0, nullptr, 0, 0, 0, nullptr};
  const int rows_upper = offsets ? static_cast<int>(a_rows) : rows_single;
  if (N % 512 == 0 && K >= 4096)
    return launch_pair<512, MODE_PLAIN_BMN>(ta, tb0, tb1, tc, ta, tb0, tb1, tc, args,
                                            rows_upper, stream);
  if (N % 256 == 0)
    return launch_pair<256, MODE_PLAIN_BMN>(ta, tb0, tb1, tc, ta, tb0, tb1, tc, args,
                                            rows_upper, stream);
  return launch_pair<128, MODE_PLAIN_BMN>(ta, tb0, tb1, tc, ta, tb0, tb1, tc, args,
                                          rows_upper, stream);
}

}  // namespace moe
