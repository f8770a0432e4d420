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
// Two kernels share one design (persistent, static round-robin over tiles):
// the CTA-pair kernel below (cta_group::2, M = 256), which every grouped GEMM
// of the layer uses, and the single-CTA kernel here, which is kept only for
// the gate/up pass that gathers its A rows from x (no permuted copy).  Roles
// of the single-CTA kernel:
//   warp 0      TMA producer: A tile 128 x 64 and B tile(s) N x 64 per stage,
//               128-byte swizzle, STAGES-deep ring of shared-memory buffers
//               (gathered rows: 16-byte cp.async by the whole warp).
//   warp 1      allocates TMEM (2 accumulators), one lane issues
//               tcgen05.mma (M=128, N=BN_ACC, K=16, bf16 x bf16 -> fp32) and
//               tcgen05.commit to release smem stages / publish accumulators.
//   warps 2-5   epilogue: tcgen05.ld the accumulator (thread = row), apply
//               SwiGLU (gate and up columns of the same output column sit in
//               the same accumulator: B rows 0-127 come from W1, 128-255 from
//               W3), round to bf16 and store the row segment.
// The TMEM accumulator is double buffered so the epilogue of tile i overlaps
// the MMAs of tile i+1.  Tile order is (group, m-tile, n-tile) with n fastest,
// so CTAs running at the same time share the A tile and one expert's weights
// in L2.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

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
constexpr int MAX_GROUPS = 257;

template <int BN_ACC>
struct GemmCfg {
  static constexpr int B_STAGE_BYTES = BN_ACC * BK * 2;
  static constexpr int STAGE_BYTES = A_STAGE_BYTES + B_STAGE_BYTES;
  static constexpr int STAGES = (196608 / STAGE_BYTES) > 8 ? 8 : (196608 / STAGE_BYTES);
  static constexpr int TMEM_COLS = 2 * BN_ACC;      // double-buffered accumulator
  // epilogue staging: per epilogue warp 32 rows x 64 bf16 (128-byte swizzle)
  static constexpr int EPI_BYTES = 4 * 32 * 128;
  static constexpr int SMEM_BYTES =
      STAGES * STAGE_BYTES + EPI_BYTES + 1024 /*align*/ + 1024 /*bars*/;
};

// Epilogue modes.
constexpr int MODE_PLAIN_BF16 = 0;    // C = A B^T, rounded to bf16
constexpr int MODE_SWIGLU_BF16 = 1;   // C = silu(A B0^T) * (A B1^T), rounded to bf16

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
};

__device__ __forceinline__ float silu_f32(float g) { return g / (1.0f + __expf(-g)); }

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

template <int BN_ACC, int MODE, bool GATHER>
__global__ void __launch_bounds__(NUM_THREADS, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                    const __grid_constant__ CUtensorMap tmB0,
                    const __grid_constant__ CUtensorMap tmB1,
                    const __grid_constant__ CUtensorMap tmC,
                    const GemmArgs args) {
  using Cfg = GemmCfg<BN_ACC>;
  constexpr int STAGES = Cfg::STAGES;
  constexpr bool SWIGLU = MODE == MODE_SWIGLU_BF16;
  constexpr int BN_OUT = SWIGLU ? BN_ACC / 2 : BN_ACC;
  constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN_ACC);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* smemA = smem;
  uint8_t* smemB = smem + STAGES * A_STAGE_BYTES;
  uint8_t* smemEpi = smem + STAGES * Cfg::STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smemEpi + Cfg::EPI_BYTES);
  uint64_t* full_bar = bars;
  uint64_t* empty_bar = bars + STAGES;
  uint64_t* tfull_bar = bars + 2 * STAGES;
  uint64_t* tempty_bar = bars + 2 * STAGES + 2;
  uint64_t* drain_bar = bars + 2 * STAGES + 4;

  __shared__ int s_off[MAX_GROUPS + 1];
  __shared__ int s_prefix[MAX_GROUPS + 1];
  __shared__ uint32_t s_tmem_base;
  __shared__ int s_abort;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_tiles = args.n_per_group / BN_OUT;
  const int G = args.offsets == nullptr ? 1 : args.num_groups;

  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull_bar[a], 1);
      mbar_init(&tempty_bar[a], 4);
    }
    mbar_init(drain_bar, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    if (!GATHER) tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB0);
    if (SWIGLU) tma_prefetch_desc(&tmB1);
    tma_prefetch_desc(&tmC);
  }
  if (warp == 1) {
    tmem_alloc(&s_tmem_base, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  pdl_wait();   // everything above touches no global memory
  if (warp == 2) build_tile_prefix(args, n_tiles, s_off, s_prefix);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem_base = s_tmem_base;
  const int total_tiles = s_prefix[G];
  volatile int* abort_flag = &s_abort;
  const int kblocks = args.K / BK;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // Lane 0 drives the ring.  With GATHER the whole warp fills the A tile
    // with 16-byte cp.async: warp instruction i copies rows 4i..4i+3 (lane
    // / 8 picks the row, lane % 8 the 16-byte chunk), written at the
    // 128-byte-swizzled position the MMA descriptor expects; each lane's
    // copies are tracked on the stage barrier by cp.async.mbarrier.arrive.
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued_mask = 0;     // stages with a load in flight at exit
    uint32_t issued_phase = 0;    // parity of that load's phase
    bool ok = true;
    for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
      const int g = find_group(s_prefix, G, tile);
      int m, n;
      tile_mn(tile - s_prefix[g], s_off[g + 1] - s_off[g], n_tiles, args.m_fastest, m, n);
      const int arow = s_off[g] + m * BM;
      const int brow = g * args.n_per_group + n * BN_OUT;
      int tok[GATHER ? 32 : 1];
      if (GATHER) {
        // rows past the group's end read a valid row (the first of the
        // tile); the epilogue never stores them
        const int rows_g = s_off[g + 1] - s_off[g];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int r = 4 * i + (lane >> 3);
          tok[i] = args.gather_rows[m * BM + r < rows_g ? arow + r : arow];
        }
      }
      for (int kb = 0; kb < kblocks; ++kb) {
        bool w_ok = true;
        if (lane == 0) w_ok = mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag);
        w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
        if (!w_ok) { ok = false; break; }
        if (GATHER) {
          const int c = lane & 7;
          uint8_t* a_tile = smemA + stage * A_STAGE_BYTES;
          const __nv_bfloat16* xa = static_cast<const __nv_bfloat16*>(args.gather_src) +
                                    kb * BK + c * 8;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int r = 4 * i + (lane >> 3);
            cp_async_16(a_tile + r * 128 + ((c ^ (r & 7)) << 4),
                        xa + static_cast<size_t>(tok[i]) * args.K);
          }
          cp_async_arrive(&full_bar[stage]);
          __syncwarp();
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(&full_bar[stage],
                                GATHER ? Cfg::B_STAGE_BYTES : Cfg::STAGE_BYTES);
          if (!GATHER)
            tma_load_2d(smemA + stage * A_STAGE_BYTES, &tmA, &full_bar[stage], kb * BK, arow);
          uint8_t* b = smemB + stage * Cfg::B_STAGE_BYTES;
          if (SWIGLU) {
            tma_load_2d(b, &tmB0, &full_bar[stage], kb * BK, brow);
            tma_load_2d(b + (BN_ACC / 2) * BK * 2, &tmB1, &full_bar[stage], kb * BK, brow);
          } else {
            tma_load_2d(b, &tmB0, &full_bar[stage], kb * BK, brow);
          }
        }
        issued_mask |= 1u << stage;
        issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
    }
    if (lane == 0) pdl_trigger();   // all loads issued: the next kernel may launch
    if (!ok && lane == 0) {
      // Let every TMA copy this CTA started land before the CTA exits.
      for (int s = 0; s < STAGES; ++s) {
        if (!(issued_mask & (1u << s))) continue;
        const uint32_t par = (issued_phase >> s) & 1u;
        const unsigned long long t0 = globaltimer_ns();
        while (!mbar_try_wait(&full_bar[s], par)) {
          if (globaltimer_ns() - t0 > kWaitLimitNs) break;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      bool issued_any = false;
      for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x, ++it) {
        const int acc = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        if (!mbar_wait(&tempty_bar[acc], acc_phase ^ 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN_ACC;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase, abort_flag)) { ok = false; break; }
          // cp.async wrote the A tile through the generic proxy; make it
          // visible to the tensor core's async-proxy reads
          if (GATHER) fence_async_shared();
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smemA + stage * A_STAGE_BYTES);
          const uint32_t b_addr = smem_u32(smemB + stage * Cfg::B_STAGE_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = smem_desc_sw128(a_addr + kk * 32);
            const uint64_t bd = smem_desc_sw128(b_addr + kk * 32);
            tc_mma_f16(d_tmem, ad, bd, IDESC, (kb | kk) != 0 ? 1u : 0u);
          }
          issued_any = true;
          tc_commit(&empty_bar[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit(&tfull_bar[acc]);
      }
      if (!ok && issued_any) {
        // Wait (bounded) for the MMAs already issued before TMEM is freed.
        tc_commit(drain_bar);
        const unsigned long long t0 = globaltimer_ns();
        while (!mbar_try_wait(drain_bar, 0)) {
          if (globaltimer_ns() - t0 > kWaitLimitNs) break;
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                   // TMEM lane quadrant of this warp
    const int row = q * 32 + lane;            // accumulator row owned by this thread
    int it = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x, ++it) {
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      // every lane waits (memory ordering); the decision is made warp-uniform
      // so the .sync.aligned TMEM loads below never run with a lane missing
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&tfull_bar[acc], acc_phase, abort_flag));
      if (!ok) break;
      tc_fence_after();
      const int g = find_group(s_prefix, G, tile);
      const int rows_g = s_off[g + 1] - s_off[g];
      int m, n;
      tile_mn(tile - s_prefix[g], rows_g, n_tiles, args.m_fastest, m, n);
      const bool valid = (m * BM + row) < rows_g;
      // a warp whose 32 rows all belong to this group stages its rows in
      // shared memory and writes them with one TMA store per 64 columns;
      // a warp that straddles the end of the group stores its valid rows
      // directly, so the next group's rows are never touched
      const bool warp_full = (m * BM + q * 32 + 32) <= rows_g;
      const int warp_row0 = s_off[g] + m * BM + q * 32;
      uint8_t* stage_buf = smemEpi + (warp - 2) * (32 * 128);
      const size_t crow_off = static_cast<size_t>(s_off[g] + m * BM + row) * args.ldc +
                              static_cast<size_t>(n) * BN_OUT;
      const uint32_t t_addr = tmem_base + acc * BN_ACC + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll 1
      for (int cb = 0; cb < BN_OUT / 64; ++cb) {
        uint32_t packed[32];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int c0 = cb * 64 + half * 32;      // first output column of this half
          uint32_t v[32];
          if (SWIGLU) {
            uint32_t u[32];
            tmem_ld16(t_addr + c0, *reinterpret_cast<uint32_t(*)[16]>(&v[0]));
            tmem_ld16(t_addr + c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&v[16]));
            tmem_ld16(t_addr + BN_OUT + c0, *reinterpret_cast<uint32_t(*)[16]>(&u[0]));
            tmem_ld16(t_addr + BN_OUT + c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&u[16]));
            tmem_ld_wait();
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
#pragma unroll
            for (int i = 0; i < 16; ++i)
              packed[half * 16 + i] =
                  pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
          }
        }
        if (warp_full) {
          if (lane == 0) bulk_wait_read_all();     // previous store has left the buffer
          __syncwarp();
          // row `lane`, 16-byte chunk c lands at chunk c ^ (lane % 8) (128-byte swizzle)
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(stage_buf + lane * 128 + ((c ^ (lane & 7)) << 4)) =
                make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2],
                           packed[4 * c + 3]);
          fence_async_shared();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmC, stage_buf, n * BN_OUT + cb * 64, warp_row0);
            bulk_commit();
          }
        } else if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(args.C) + crow_off +
                                                cb * 64);
#pragma unroll
          for (int c = 0; c < 8; ++c)
            dst[c] = make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2],
                                packed[4 * c + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty_bar[acc]);
    }
    if (lane == 0) bulk_wait_all();            // this warp's TMA stores are complete
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && s_abort) atomicOr(args.status, kDevTimeout);
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
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

template <int BN_ACC, int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                         const __grid_constant__ CUtensorMap tmB0,
                         const __grid_constant__ CUtensorMap tmB1,
                         const __grid_constant__ CUtensorMap tmC, const GemmArgs args) {
  using Cfg = PairCfg<BN_ACC>;
  constexpr int STAGES = Cfg::STAGES;
  constexpr bool SWIGLU = MODE == MODE_SWIGLU_BF16;
  constexpr int BN_OUT = SWIGLU ? BN_ACC / 2 : BN_ACC;
  constexpr int NSUB = Cfg::NSUB;
  constexpr int NACC = Cfg::NACC;
  constexpr uint32_t IDESC = idesc_bf16_f32(BM2, Cfg::N_MMA);

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
  const int n_tiles = args.n_per_group / BN_OUT;
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
    if (SWIGLU) tma_prefetch_desc(&tmB1);
    tma_prefetch_desc(&tmC);
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
  const int total_tiles = s_prefix[G];
  volatile int* abort_flag = &s_abort;
  const int kblocks = args.K / BK;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, issued_mask = 0, issued_phase = 0;
      bool ok = true;
      for (int tile = pair; tile < total_tiles && ok; tile += npairs) {
        const int g = find_group(s_prefix, G, tile);
        int m, n;
        tile_mn<BM2>(tile - s_prefix[g], s_off[g + 1] - s_off[g], n_tiles, args.m_fastest, m, n);
        const int arow = s_off[g] + m * BM2 + static_cast<int>(rank) * BM;
        const int brow = SWIGLU ? g * args.n_per_group + n * BN_OUT
                                : g * args.n_per_group + n * BN_OUT + static_cast<int>(rank) * (BN_ACC / 2);
        const CUtensorMap* mb = (SWIGLU && rank == 1) ? &tmB1 : &tmB0;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
          if (rank == 0) mbar_arrive_expect_tx(&full_bar[stage], 2 * Cfg::STAGE_BYTES);
          tma_load_2d_pair(smemA + stage * A_STAGE_BYTES, &tmA, &full_bar[stage], kb * BK, arow);
          tma_load_2d_pair(smemB + stage * Cfg::B_HALF_BYTES, mb, &full_bar[stage], kb * BK, brow);
          issued_mask |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
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
            for (int sub = 0; sub < NSUB; ++sub)   // sub-tile: B rows [128 sub, 128 sub + 128)
              tc_mma_f16_pair(d_tmem + sub * Cfg::N_MMA, smem_desc_sw128(a_addr + kk * 32),
                              smem_desc_sw128(b_addr + sub * (Cfg::N_MMA / 2) * 128 + kk * 32),
                              IDESC, (kb | kk) != 0 ? 1u : 0u);
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
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int row = q * 32 + lane;
    int it = 0;
    for (int tile = pair; tile < total_tiles; tile += npairs, ++it) {
      const int acc = it % NACC;
      const uint32_t acc_phase = (it / NACC) & 1;
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&tfull_bar[acc], acc_phase, abort_flag));
      if (!ok) break;
      tc_fence_after();
      const int g = find_group(s_prefix, G, tile);
      const int rows_g = s_off[g + 1] - s_off[g];
      int m, n;
      tile_mn<BM2>(tile - s_prefix[g], rows_g, n_tiles, args.m_fastest, m, n);
      const int r0 = m * BM2 + static_cast<int>(rank) * BM;   // first row (in group) of this CTA
      const bool valid = (r0 + row) < rows_g;
      const bool warp_full = (r0 + q * 32 + 32) <= rows_g;
      const int warp_row0 = s_off[g] + r0 + q * 32;
      uint8_t* stage_buf = smemEpi + (warp - 2) * (32 * 128);
      const size_t crow_off = static_cast<size_t>(s_off[g] + r0 + row) * args.ldc;
      const uint32_t t_addr = tmem_base + acc * BN_ACC + (static_cast<uint32_t>(q * 32) << 16);
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
        uint32_t packed[32];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int c0 = acol + half * 32;
          uint32_t v[32];
          if (SWIGLU) {
            uint32_t u[32];
            constexpr int UP = Cfg::N_MMA / 2;   // up columns follow the gate columns
            tmem_ld16(t_addr + c0, *reinterpret_cast<uint32_t(*)[16]>(&v[0]));
            tmem_ld16(t_addr + c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&v[16]));
            tmem_ld16(t_addr + UP + c0, *reinterpret_cast<uint32_t(*)[16]>(&u[0]));
            tmem_ld16(t_addr + UP + c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&u[16]));
            tmem_ld_wait();
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
#pragma unroll
            for (int i = 0; i < 16; ++i)
              packed[half * 16 + i] =
                  pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
          }
        }
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
            tma_store_2d(&tmC, stage_buf, ocol, warp_row0);
            bulk_commit();
          }
        } else if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(args.C) + crow_off +
                                                ocol);
#pragma unroll
          for (int c = 0; c < 8; ++c)
            dst[c] = make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2],
                                packed[4 * c + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_rank0(&tempty_bar[acc]);
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
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

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
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

template <int BN_ACC, int MODE, bool GATHER = false>
cudaError_t launch(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                   const CUtensorMap& c, const GemmArgs& args, int rows_upper,
                   cudaStream_t stream) {
  using Cfg = GemmCfg<BN_ACC>;
  constexpr int BN_OUT = MODE == MODE_SWIGLU_BF16 ? BN_ACC / 2 : BN_ACC;
  auto kern = grouped_gemm_kernel<BN_ACC, MODE, GATHER>;
  static unsigned long long attr_done = 0;   // one bit per device (attribute is per device)
  int dev = 0;
  cudaGetDevice(&dev);
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(attr_done & bit)) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Cfg::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_done |= bit;
  }
  const int G = args.offsets == nullptr ? 1 : args.num_groups;
  // m-fastest order once one group's weights (B rows x K, both halves for
  // SwiGLU) exceed 32 MB, a quarter of the L2
  GemmArgs a2 = args;
  const double b_bytes = static_cast<double>(BN_OUT == BN_ACC ? args.n_per_group
                                                              : 2 * args.n_per_group) *
                         args.K * 2.0;
  a2.m_fastest = b_bytes > 32.0 * 1024 * 1024 ? 1 : 0;
  const long long m_tiles_upper = (rows_upper + BM - 1) / BM + (G > 1 ? G : 0);
  const long long tiles_upper = m_tiles_upper * (args.n_per_group / BN_OUT);
  if (tiles_upper <= 0) return cudaSuccess;
  const int grid = static_cast<int>(tiles_upper < num_sms() ? tiles_upper : num_sms());
  return launch_pdl(kern, dim3(grid), dim3(NUM_THREADS), Cfg::SMEM_BYTES, stream, a, b0, b1, c,
                    a2);
}

template <int BN_ACC, int MODE>
cudaError_t launch_pair(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                        const CUtensorMap& c, const GemmArgs& args, int rows_upper,
                        cudaStream_t stream) {
  using Cfg = PairCfg<BN_ACC>;
  constexpr int BN_OUT = MODE == MODE_SWIGLU_BF16 ? BN_ACC / 2 : BN_ACC;
  auto kern = grouped_gemm_pair_kernel<BN_ACC, MODE>;
  static unsigned long long attr_done = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(attr_done & bit)) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Cfg::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_done |= bit;
  }
  const int G = args.offsets == nullptr ? 1 : args.num_groups;
  GemmArgs a2 = args;
  const double b_bytes = static_cast<double>(BN_OUT == BN_ACC ? args.n_per_group
                                                              : 2 * args.n_per_group) *
                         args.K * 2.0;
  a2.m_fastest = b_bytes > 32.0 * 1024 * 1024 ? 1 : 0;
  const long long m_tiles_upper = (rows_upper + BM2 - 1) / BM2 + (G > 1 ? G : 0);
  const long long tiles_upper = m_tiles_upper * (args.n_per_group / BN_OUT);
  if (tiles_upper <= 0) return cudaSuccess;
  const int max_pairs = num_sms() / 2;
  const int pairs = static_cast<int>(tiles_upper < max_pairs ? tiles_upper : max_pairs);
  return launch_pdl(kern, dim3(2 * pairs), dim3(NUM_THREADS), Cfg::SMEM_BYTES, stream, a, b0, b1,
                    c, a2);
}

}  // namespace

// h[r] = silu(A[r] W1[g]^T) * (A[r] W3[g]^T), bf16 out.
cudaError_t grouped_swiglu_gateup_bf16(const void* A, int64_t a_rows, const int32_t* offsets,
                                       int num_groups, int rows_single, const void* W1,
                                       const void* W3, int F, int K, void* H, uint32_t* status,
                                       cudaStream_t stream) {
  CUtensorMap ta, tb0, tb1, tc;
  const int64_t b_rows = static_cast<int64_t>(offsets ? num_groups : 1) * F;
  const int64_t c_rows = offsets ? a_rows : rows_single;
  // 256 output columns per tile (512 accumulator columns) when F allows
  const bool wide = F % 256 == 0;
  const int bh = wide ? 256 : 128;   // B rows each CTA of the pair loads
  if (!make_map(&ta, A, a_rows, K, BM) || !make_map(&tb0, W1, b_rows, K, bh) ||
      !make_map(&tb1, W3, b_rows, K, bh) || !make_map(&tc, H, c_rows, F, 32))
    return cudaErrorInvalidValue;
  GemmArgs args{offsets, num_groups, rows_single, F, K, H, F, status, nullptr, nullptr, 0};
  const int rows_upper = offsets ? static_cast<int>(a_rows) : rows_single;
  if (wide) return launch_pair<512, MODE_SWIGLU_BF16>(ta, tb0, tb1, tc, args, rows_upper, stream);
  return launch_pair<256, MODE_SWIGLU_BF16>(ta, tb0, tb1, tc, args, rows_upper, stream);
}

// Gate/up pass whose A rows are gathered from X [x_rows, K]: output row r
// (expert-contiguous order, r < R) reads X[rows[r]].  H is [R, F].
cudaError_t grouped_swiglu_gateup_gather_bf16(const void* X, int64_t x_rows, const int32_t* rows,
                                              int64_t R, const int32_t* offsets, int num_groups,
                                              const void* W1, const void* W3, int F, int K,
                                              void* H, uint32_t* status, cudaStream_t stream) {
  CUtensorMap tb0, tb1, tc;
  const int64_t b_rows = static_cast<int64_t>(num_groups) * F;
  (void)x_rows;
  if (!make_map(&tb0, W1, b_rows, K, 128) || !make_map(&tb1, W3, b_rows, K, 128) ||
      !make_map(&tc, H, R, F, 32))
    return cudaErrorInvalidValue;
  GemmArgs args{offsets, num_groups, 0, F, K, H, F, status, rows, X, 0};
  // tmA is unused in gather mode (A comes through cp.async)
  return launch<256, MODE_SWIGLU_BF16, true>(tb0, tb0, tb1, tc, args, static_cast<int>(R), stream);
}

// Y[r] = A[r] W2[g]^T, bf16 out; N = output columns per group.
cudaError_t grouped_down_bf16(const void* A, int64_t a_rows, const int32_t* offsets,
                              int num_groups, int rows_single, const void* W2, int N, int K,
                              void* Y, uint32_t* status, cudaStream_t stream) {
  CUtensorMap ta, tb, tc;
  const int64_t b_rows = static_cast<int64_t>(offsets ? num_groups : 1) * N;
  const int64_t c_rows = offsets ? a_rows : rows_single;
  const int bn = (N % 512 == 0) ? 512 : (N % 256 == 0) ? 256 : 128;
  // each CTA of the pair loads half of the B tile
  if (!make_map(&ta, A, a_rows, K, BM) || !make_map(&tb, W2, b_rows, K, bn / 2) ||
      !make_map(&tc, Y, c_rows, N, 32))
    return cudaErrorInvalidValue;
  GemmArgs args{offsets, num_groups, rows_single, N, K, Y, N, status, nullptr, nullptr, 0};
  const int rows_upper = offsets ? static_cast<int>(a_rows) : rows_single;
  if (bn == 512)
    return launch_pair<512, MODE_PLAIN_BF16>(ta, tb, tb, tc, args, rows_upper, stream);
  if (bn == 256)
    return launch_pair<256, MODE_PLAIN_BF16>(ta, tb, tb, tc, args, rows_upper, stream);
  return launch_pair<128, MODE_PLAIN_BF16>(ta, tb, tb, tc, args, rows_upper, stream);
}


}  // namespace moe
