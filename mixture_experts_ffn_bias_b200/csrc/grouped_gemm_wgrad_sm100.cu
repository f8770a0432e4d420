// K-grouped GEMM on tcgen05 tensor cores: the weight gradients of the
// grouped experts.
//
// For every group (expert) g:   C_g [M, N] = A_g^T B_g,   bf16 in, fp32
// accumulate in TMEM, bf16 out, C stored as [G, M, N].
// A_g and B_g are the rows [off[g], off[g+1]) of A [R, lda] (columns
// [a_col0, a_col0 + M)) and B [R, ldb] (columns [b_col0, b_col0 + N)): the
// activations of the expert's rows as the forward and backward keep them, so
// the reduction dimension (rows) is the strided one and both operands are
// read MN-major, with no transposed copy.  For the down projection
// dW2[g] = dY_g^T H_g (A = dY, B = H); for the gate/up projections
// dW1[g] = dG_g^T X_g and dW3[g] = dU_g^T X_g (A = [dG | dU] from column 0
// or F, B = X's rows in expert order).  A group's rows start anywhere; its
// last 64-row k-block may reach into the next group's rows, which are zeroed
// in the A tile in shared memory before the MMAs read it, so they add
// nothing.  An expert with no rows gets C_g = 0 (written by the epilogue
// without touching the accumulator ring).
//
// Structure (one CTA per SM, persistent over (g, m, n) tiles, n fastest):
//   warp 0      TMA producer: A tile 64 k x 128 m (two 64-column boxes),
//               B tile 64 k x BN n per stage, 128-byte swizzle
//   warp 1      TMEM allocation; zeroes the rows past a group in its last
//               A tile; one lane issues tcgen05.mma (M = 128, N = BN, K =
//               16 per instruction, both operands MN-major) into a
//               double-buffered accumulator
//   warps 2..5  epilogue: TMEM -> registers -> bf16, staged 32 rows x 64
//               columns per warp in shared memory, TMA tensor stores
// Every wait is bounded; a wait that gives up aborts the CTA and sets the
// timeout bit of the status word.
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

constexpr int WBM = 128;
constexpr int WBK = 64;
constexpr int W_A_BYTES = WBM * WBK * 2;
constexpr int W_THREADS = 192;
constexpr int W_MAX_GROUPS = 257;

template <int BN>
struct WCfg {
  static constexpr int B_BYTES = BN * WBK * 2;
  static constexpr int STAGE_BYTES = W_A_BYTES + B_BYTES;
  static constexpr int STAGES = (196608 / STAGE_BYTES) > 8 ? 8 : (196608 / STAGE_BYTES);
  static constexpr int TMEM_COLS = 2 * BN;
  // epilogue staging: per epilogue warp 32 rows x 64 bf16 (128-byte swizzle)
  static constexpr int EPI_BYTES = 4 * 32 * 128;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_BYTES + 1024 + 1024;
};

struct WgradArgs {
  const int32_t* offsets;  // [G+1] row offsets of the groups, or null: one group of rows_single
  int rows_single;
  int G, M, N;
  int a_col0, b_col0;      // first column of A and of B taken
  __nv_bfloat16* C;        // [G, M, N]
  uint32_t* status;
};

constexpr int W_BOX = 64 * 128;   // one 64-column x 64-row box of an MN-major operand

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

template <int BN>
__global__ void __launch_bounds__(W_THREADS, 1)
wgrad_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
             const __grid_constant__ CUtensorMap tmC, const WgradArgs args) {
  using Cfg = WCfg<BN>;
  constexpr int STAGES = Cfg::STAGES;
  constexpr uint32_t IDESC = idesc_bf16_f32(WBM, BN, true, true);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * W_A_BYTES;
  uint8_t* sEpi = smem + STAGES * Cfg::STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sEpi + Cfg::EPI_BYTES);
  uint64_t* full_bar = bars;
  uint64_t* empty_bar = bars + STAGES;
  uint64_t* tfull_bar = bars + 2 * STAGES;
  uint64_t* tempty_bar = bars + 2 * STAGES + 2;
  uint64_t* drain_bar = bars + 2 * STAGES + 4;
  __shared__ int s_off[W_MAX_GROUPS + 1];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int MT = args.M / WBM, NT = args.N / BN;
  const int total = args.G * MT * NT;

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
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmC);
  }
  if (warp == 1) {
    tmem_alloc(&s_tmem, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  pdl_wait();   // everything above touches no global memory
  if (warp == 2) {
    if (args.offsets)
      for (int i = lane; i <= args.G; i += 32) s_off[i] = args.offsets[i];
    else if (lane == 0) {
      s_off[0] = 0;
      s_off[1] = args.rows_single;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  volatile int* abort_flag = &s_abort;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, issued_mask = 0, issued_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        const int g = tile / (MT * NT);
        const int rem = tile - g * MT * NT;
        const int m = rem / NT, n = rem - (rem / NT) * NT;
        const int k0 = s_off[g], kbs = (s_off[g + 1] - k0 + WBK - 1) / WBK;
        for (int kb = 0; kb < kbs; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&full_bar[stage], Cfg::STAGE_BYTES);
          const int krow = k0 + kb * WBK;
#pragma unroll
          for (int j = 0; j < WBM / 64; ++j)
            tma_load_2d(sA + stage * W_A_BYTES + j * W_BOX, &tmA, &full_bar[stage],
                        args.a_col0 + m * WBM + j * 64, krow);
#pragma unroll
          for (int j = 0; j < BN / 64; ++j)
            tma_load_2d(sB + stage * Cfg::B_BYTES + j * W_BOX, &tmB, &full_bar[stage],
                        args.b_col0 + n * BN + j * 64, krow);
          issued_mask |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      pdl_trigger();
      if (!ok) {
        for (int s = 0; s < STAGES; ++s) {
          if (!(issued_mask & (1u << s))) continue;
          const unsigned long long t0 = globaltimer_ns();
          while (!mbar_try_wait(&full_bar[s], (issued_phase >> s) & 1u))
            if (globaltimer_ns() - t0 > kWaitLimitNs) break;
        }
      }
    }
  } else if (warp == 1) {
    // the whole warp follows the tiles: lane 0 issues the MMAs, all lanes
    // zero the rows past a group in its last A tile
    int stage = 0, it = 0;
    uint32_t phase = 0;
    bool ok = true, issued = false;
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
      const int g = tile / (MT * NT);
      const int rows_g = s_off[g + 1] - s_off[g];
      const int kbs = (rows_g + WBK - 1) / WBK;
      if (kbs == 0) continue;   // empty group: the epilogue writes zeros, no accumulator
      const int acc = it & 1;
      ok = __all_sync(0xffffffffu,
                      mbar_wait(&tempty_bar[acc], ((it >> 1) & 1) ^ 1u, abort_flag));
      if (!ok) break;
      tc_fence_after();
      const uint32_t d = tmem + acc * BN;
      for (int kb = 0; kb < kbs; ++kb) {
        ok = __all_sync(0xffffffffu, mbar_wait(&full_bar[stage], phase, abort_flag));
        if (!ok) break;
        const int valid = rows_g - kb * WBK;   // rows of this k-block in the group
        if (valid < WBK) {
          // rows [valid, 64) of both A boxes belong to the next group (or
          // lie past the tensor): zero them, 16 bytes per lane per store;
          // each row of a box is 128 contiguous bytes whatever the swizzle
          uint8_t* a_st = sA + stage * W_A_BYTES;
          const int per_box = (WBK - valid) * 8;
          for (int i = lane; i < 2 * per_box; i += 32) {
            const int box = i / per_box, c = i - box * per_box;
            *reinterpret_cast<uint4*>(a_st + box * W_BOX + valid * 128 + c * 16) =
                make_uint4(0u, 0u, 0u, 0u);
          }
          fence_async_shared();   // visible to the tensor cores' reads
        }
        __syncwarp();
        if (lane == 0) {
          tc_fence_after();
          const uint32_t a = smem_u32(sA + stage * W_A_BYTES);
          const uint32_t b = smem_u32(sB + stage * Cfg::B_BYTES);
#pragma unroll
          for (int kk = 0; kk < WBK / 16; ++kk)
            tc_mma_f16(d, smem_desc_sw128_mn(a + kk * 16 * 128, W_BOX),
                       smem_desc_sw128_mn(b + kk * 16 * 128, W_BOX), IDESC,
                       (kb | kk) != 0 ? 1u : 0u);
          tc_commit(&empty_bar[stage]);
        }
        issued = true;
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
      if (lane == 0) tc_commit(&tfull_bar[acc]);
      ++it;
    }
    if (!ok && issued && lane == 0) {
      tc_commit(drain_bar);
      const unsigned long long t0 = globaltimer_ns();
      while (!mbar_try_wait(drain_bar, 0))
        if (globaltimer_ns() - t0 > kWaitLimitNs) break;
    }
    __syncwarp();
  } else {
    const int q = warp & 3;
    const int row = q * 32 + lane;
    // the weight gradients are not read again here: stored evict-first, so
    // the L2 keeps the activation tiles other CTAs are about to re-read
    const uint64_t c_policy = l2_policy_evict_first();
    int it = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      const int g = tile / (MT * NT);
      const int rem = tile - g * MT * NT;
      const int m = rem / NT, n = rem - (rem / NT) * NT;
      uint4* dst = reinterpret_cast<uint4*>(
          args.C + (static_cast<size_t>(g) * args.M + m * WBM + row) * args.N +
          static_cast<size_t>(n) * BN);
      if (s_off[g + 1] == s_off[g]) {   // empty group: C_g = 0, no accumulator used
        for (int c = 0; c < BN / 8; ++c) dst[c] = make_uint4(0u, 0u, 0u, 0u);
        continue;
      }
      const int acc = it & 1;
      const bool ok =
          __all_sync(0xffffffffu, mbar_wait(&tfull_bar[acc], (it >> 1) & 1, abort_flag));
      ++it;
      if (!ok) break;
      tc_fence_after();
      const uint32_t taddr = tmem + acc * BN + (static_cast<uint32_t>(q * 32) << 16);
      // Each warp stages its 32 rows x 64 columns in shared memory with the
      // 128-byte swizzle and writes them with one TMA tensor store.
      uint8_t* stage_buf = sEpi + (warp - 2) * (32 * 128);
      const int crow0 = g * args.M + m * WBM + q * 32;
#pragma unroll 1
      for (int cb = 0; cb < BN / 64; ++cb) {
        uint32_t p[32];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t v[32];
          tmem_ld16(taddr + cb * 64 + half * 32, *reinterpret_cast<uint32_t(*)[16]>(&v[0]));
          tmem_ld16(taddr + cb * 64 + half * 32 + 16, *reinterpret_cast<uint32_t(*)[16]>(&v[16]));
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i)
            p[half * 16 + i] = pack2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
        }
        if (lane == 0) bulk_wait_read_all();     // the previous store has left the buffer
        __syncwarp();
        // row `lane`, 16-byte chunk c lands at chunk c ^ (lane % 8)
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(stage_buf + lane * 128 + ((c ^ (lane & 7)) << 4)) =
              make_uint4(p[4 * c], p[4 * c + 1], p[4 * c + 2], p[4 * c + 3]);
        fence_async_shared();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d_hint(&tmC, stage_buf, n * BN + cb * 64, crow0, c_policy);
          bulk_commit();
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
    tmem_dealloc(tmem, Cfg::TMEM_COLS);
  }
}

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                              const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                              const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                              CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// Looked up once per process; the initialisation of a function-local
// static is thread-safe.
EncodeFn encode() {
  static const EncodeFn fn = []() -> EncodeFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeFn>(p);
    return nullptr;
  }();
  return fn;
}

// [rows, cols] bf16, boxes of box_rows x 64 with the 128-byte swizzle.
bool map_rows(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_rows) {
  EncodeFn enc = encode();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(WBK), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

template <int BN>
cudaError_t launch_wgrad(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tc,
                         const WgradArgs& a, cudaStream_t stream) {
  using Cfg = WCfg<BN>;
  auto kern = wgrad_kernel<BN>;
  static std::atomic<unsigned long long> attr_done{0};
  int dev = 0;
  cudaGetDevice(&dev);
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(attr_done.load(std::memory_order_acquire) & bit)) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_done.fetch_or(bit, std::memory_order_acq_rel);
  }
  int sms = 0;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (sms <= 0) sms = 148;
  const long long tiles = static_cast<long long>(a.G) * (a.M / WBM) * (a.N / BN);
  if (tiles <= 0) return cudaSuccess;
  const int grid = static_cast<int>(tiles < sms ? tiles : sms);
  return launch_pdl(kern, dim3(grid), dim3(W_THREADS), Cfg::SMEM_BYTES, stream, ta, tb, tc, a);
}

}  // namespace

cudaError_t grouped_wgrad_bf16(const void* A, int lda, int a_col0, const void* B, int ldb,
                               int b_col0, int64_t rows, const int32_t* offsets, int G, int M,
                               int N, void* C, uint32_t* status, cudaStream_t stream) {
  if (M % WBM || N % 128 || G > W_MAX_GROUPS - 1 || a_col0 % 64 || b_col0 % 64 ||
      a_col0 + M > lda || b_col0 + N > ldb || (offsets == nullptr && G != 1) ||
      rows > 0x7fffffff)
    return cudaErrorInvalidValue;
  const int bn = (N % 256 == 0) ? 256 : 128;
  CUtensorMap ta, tb, tc;
  if (!map_rows(&ta, A, rows, lda, WBK) || !map_rows(&tb, B, rows, ldb, WBK) ||
      !map_rows(&tc, C, static_cast<int64_t>(G) * M, N, 32))
    return cudaErrorInvalidValue;
  WgradArgs a{offsets, static_cast<int>(rows), G, M, N, a_col0, b_col0,
              static_cast<__nv_bfloat16*>(C), status};
  if (bn == 256) return launch_wgrad<256>(ta, tb, tc, a, stream);
  return launch_wgrad<128>(ta, tb, tc, a, stream);
}

}  // namespace moe
