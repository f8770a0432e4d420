// Router logits on tcgen05 tensor cores with chunked accumulation.
//
// logits[t, e] = x[t] . Wr[e]  (the fp32 router linear of SigmoidRouter in
// the "moe-200m-qwen3-100b" README, "Per-layer numerics": routing in fp32).
//
// bf16 x bf16 products are exact in fp32, so all the error of a tensor-core
// logit is in the accumulation.  Accumulating the whole K (2048-5120) in one
// TMEM accumulator gave errors up to ~1e-5 on unit-scale logits; here each
// 128-wide K chunk is accumulated in a fresh TMEM slot (8 MMAs on a partial of
// magnitude ~0.2) and the epilogue warps add the chunk partials into fp32
// registers while the MMAs of the next chunks run.  This keeps the logit
// error in the low 1e-6 range, far inside the router's re-decision margin.
//
// With up to 128 experts and top-k <= 8 the routing decision is taken in the
// same kernel (fused select): the epilogue thread that owns a token's row holds
// all of its logits in registers, forms the gate statistics and the selection
// keys and picks the top-(k+1) keys (descending, ties to the lower expert id)
// from per-group best keys, re-scanning only the winning group each round
// (the logits kept in the thread's shared-memory column).  A token whose
// picked keys hold two keys
// closer than kRefineMargin is not decided here: it is listed together with
// its candidate experts (every expert whose key is within the margin of the
// (k+1)-th pick), and router_refine_kernel decides it on exact logits.
// Otherwise the logits are written out and router_select_fast_kernel decides.
//
// Warp roles (persistent over 128-token tiles):
//   warp 0        TMA: x tile 128 x 64 and Wr tile NPAD x 64 per stage
//   warp 1        TMEM allocation; one lane issues tcgen05.mma into a ring of
//                 NSLOT accumulator slots (one slot per K chunk)
//   warps 2..     epilogue: one accumulator row per thread, NPAD <= 128
//                 columns per warpgroup (two warpgroups for NPAD = 256)
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

constexpr int RBM = 128;
constexpr int RBK = 64;
constexpr int KCH = 2;                       // k-blocks per accumulation chunk
constexpr int R_A_BYTES = RBM * RBK * 2;

constexpr int KMAX_FUSED = 8;
constexpr int PICKS = KMAX_FUSED + 2;        // a part's picks (k + 1 at most) and an end mark
constexpr int kSelectParts = 4;              // fused select over 128 experts: 4 x 32 keys

template <int NPAD, bool FUSED = false>
struct RCfg {
  // Epilogue warpgroups: each holds NPAD / EPI_WG accumulator columns of
  // every row.  The fused select over 128 experts splits a token's keys
  // between kSelectParts threads, which divides the serial per-thread work
  // and gives each SM sub-partition more warps to interleave; the first
  // warpgroup merges the partial rankings.
  static constexpr int EPI_WG = (FUSED && NPAD == 128) ? kSelectParts : (NPAD > 128 ? 2 : 1);
  static constexpr int COLS = NPAD / EPI_WG;           // columns per epilogue thread
  static constexpr int THREADS = 64 + 128 * EPI_WG;
  static constexpr int B_BYTES = NPAD * RBK * 2;
  static constexpr int STAGE_BYTES = R_A_BYTES + B_BYTES;
  // fused select keeps each token's logits in a shared-memory column, and
  // each warpgroup's partial ranking (values and ids) in two more
  static constexpr int LOGIT_BYTES = FUSED ? NPAD * 128 * 4 : 0;
  static constexpr int PICK_BYTES = FUSED ? EPI_WG * PICKS * 128 * 8 : 0;
  static constexpr int STAGE_BUDGET = 226304 - LOGIT_BYTES - PICK_BYTES;   // of 227 KB
  static constexpr int STAGES = (STAGE_BUDGET / STAGE_BYTES) > 8 ? 8 : (STAGE_BUDGET / STAGE_BYTES);
  static constexpr int NSLOT = (512 / NPAD) > 8 ? 8 : (512 / NPAD);
  static constexpr int TMEM_RAW = NSLOT * NPAD;
  static constexpr int TMEM_COLS = TMEM_RAW <= 32 ? 32 : TMEM_RAW <= 64 ? 64
                                   : TMEM_RAW <= 128 ? 128 : TMEM_RAW <= 256 ? 256 : 512;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + LOGIT_BYTES + PICK_BYTES + 1024 + 1024;
};

// TMA tile load with an L2 eviction-priority policy (the router's x tiles
// are marked evict-last, so the dispatch scatter that re-reads x right after
// the router finds most of it in L2).
__device__ __forceinline__ uint64_t l2_evict_last_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ void tma_load_2d_hint(void* dst, const CUtensorMap* map,
                                                 uint64_t* bar, int32_t x, int32_t y,
                                                 uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)),
        "r"(x), "r"(y), "l"(policy)
      : "memory");
}

struct RouterOut {
  float* logits;                 // unfused: [T, E] fp32
  const float* offset;           // fused: per-expert logit offset or null
  const float* bias;             // fused: selection bias or null
  int k, gate, renorm;
  int32_t* topk_idx;             // fused outputs
  float* topk_w;
  int32_t* refine_count;
  int32_t* refine_list;          // [T] listed tokens
  int32_t* refine_cand;          // [T, kRefineCand] candidate experts (-1 pad, -2 = all)
  uint32_t* status;
};

// Fused select, part 1, run by every epilogue thread for its token over the
// experts [base, base + COLS) whose logits it holds in acc[] (i < E only).
// The logits (with the per-expert offset) go to the token's shared-memory
// column s_log[e * 128], acc[] becomes the selection keys (logit + bias),
// and the best min(rounds, experts here) keys in (descending key, ascending
// id) order go to pv/pi[j * 128] with an end mark after them.  Returns the
// largest logit of the part.
//
// One thread owns a (token, part) and only a few warps run this per SM, so
// the code is written for instruction-level parallelism: no branches inside
// the loops (even a warp-uniform branch splits an unrolled loop into blocks
// that cannot be interleaved), selects instead of short-circuit conditions,
// four partial maxima and sums, loads kept apart from stores.  The ranking
// splits the part into NG groups of GS consecutive ids, each holding its
// best key not yet picked; a round takes the best group head and re-scans
// only that group (keys re-formed from the logit column and the bias: the
// same fp32 sums as acc[]).
template <int COLS>
__device__ __forceinline__ float route_part(float (&acc)[COLS], float* s_log, const float* s_off,
                                            const float* s_bias, int base, int E, int rounds,
                                            float* pv, int* pi) {
  constexpr int NONE = 0x7fffffff;
  float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
  for (int i = 0; i < COLS; i += 4) {
    const float4 f = *reinterpret_cast<const float4*>(s_off + base + i);
    const float ov[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float l = base + i + q < E ? acc[i + q] + ov[q] : -INFINITY;
      acc[i + q] = l;
      mx[q] = fmaxf(mx[q], l);
    }
  }
#pragma unroll
  for (int i = 0; i < COLS; ++i) s_log[(base + i) * 128] = acc[i];
#pragma unroll
  for (int i = 0; i < COLS; i += 4) {
    const float4 f = *reinterpret_cast<const float4*>(s_bias + base + i);
    const float bv[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
    for (int q = 0; q < 4; ++q)
      acc[i + q] = base + i + q < E ? acc[i + q] + bv[q] : -INFINITY;
  }
  const float m = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
  constexpr int GS = COLS >= 64 ? 8 : 4;
  constexpr int NG = COLS / GS;
  float gv[NG];
  int gi[NG];
#pragma unroll
  for (int g = 0; g < NG; ++g) {
    gv[g] = acc[g * GS];
    gi[g] = base + g * GS;
#pragma unroll
    for (int s = 1; s < GS; ++s) {
      const bool take = acc[g * GS + s] > gv[g];
      gv[g] = take ? acc[g * GS + s] : gv[g];
      gi[g] = take ? base + g * GS + s : gi[g];
    }
    gi[g] = base + g * GS < E ? gi[g] : NONE;   // a group wholly past E holds nothing
  }
  const int here = E - base < COLS ? (E - base > 0 ? E - base : 0) : COLS;
  const int n = rounds < here ? rounds : here;
#pragma unroll 1
  for (int j = 0; j < n; ++j) {
    // groups are in id order, so on equal heads the earlier group wins
    float bv = gv[0];
    int bi = gi[0], bg = 0;
#pragma unroll
    for (int g = 1; g < NG; ++g) {
      const bool take = (gi[g] != NONE) & ((bi == NONE) | (gv[g] > bv));
      bv = take ? gv[g] : bv;
      bi = take ? gi[g] : bi;
      bg = take ? g : bg;
    }
    pv[j * 128] = bv;
    pi[j * 128] = bi;
    float vv[GS];
#pragma unroll
    for (int s = 0; s < GS; ++s) {
      const int i = base + bg * GS + s;
      vv[s] = i < E ? s_log[i * 128] + s_bias[i] : -INFINITY;
    }
    float nv = -INFINITY;
    int ni = NONE;
#pragma unroll
    for (int s = 0; s < GS; ++s) {
      const int i = base + bg * GS + s;
      const bool after = (vv[s] < bv) | ((vv[s] == bv) & (i > bi));
      const bool take = (i < E) & after & ((vv[s] > nv) | (ni == NONE));
      nv = take ? vv[s] : nv;
      ni = take ? i : ni;
    }
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      gv[g] = g == bg ? nv : gv[g];
      gi[g] = g == bg ? ni : gi[g];
    }
  }
  pv[n * 128] = -INFINITY;   // end mark
  pi[n * 128] = NONE;
  return m;
}

// Fused select, part 2, for one token: merge the NP partial rankings (part p
// holds lower expert ids than part p + 1, so equal keys take the earlier
// part) into the top-(k+1) keys, then either list the token for exact
// re-decision (two of those keys closer than kRefineMargin) with its
// candidate experts, or write its k experts and weights.  m_part[128 p]:
// the parts' largest logits.
template <int NP>
__device__ __forceinline__ void route_finish(const float* pv, const int* pi, int pstride,
                                             const float* m_part, const float* s_log,
                                             const float* s_bias, int E, int t,
                                             const RouterOut& o) {
  constexpr int NONE = 0x7fffffff;
  const int rounds = o.k < E ? o.k + 1 : o.k;
  int head[NP];
#pragma unroll
  for (int p = 0; p < NP; ++p) head[p] = 0;
  int sid[KMAX_FUSED];
  float prev = 0.f, min_gap = INFINITY;
#pragma unroll
  for (int j = 0; j < KMAX_FUSED + 1; ++j) {
    if (j < rounds) {
      float bv = pv[head[0] * 128];
      int bi = pi[head[0] * 128], bp = 0;
#pragma unroll
      for (int p = 1; p < NP; ++p) {
        const float v = pv[p * pstride + head[p] * 128];
        const int i = pi[p * pstride + head[p] * 128];
        const bool take = (i != NONE) & ((bi == NONE) | (v > bv));
        bv = take ? v : bv;
        bi = take ? i : bi;
        bp = take ? p : bp;
      }
#pragma unroll
      for (int p = 0; p < NP; ++p) head[p] += p == bp ? 1 : 0;
      min_gap = j > 0 ? fminf(min_gap, prev - bv) : min_gap;
      prev = bv;
      if (j < KMAX_FUSED) sid[j] = bi;
    }
  }
  if (min_gap < kRefineMargin) {
    // list the token with its candidate experts: every expert whose key is
    // within the margin of the last pick (the exact top-k is among them);
    // softmax without renormalisation needs all exact logits
    const int slot = atomicAdd(o.refine_count, 1);
    o.refine_list[slot] = t;
    int32_t* cand = o.refine_cand + static_cast<size_t>(slot) * kRefineCand;
    const float lo = prev - kRefineMargin;
    uint32_t msk[4];   // E <= 128 here
    int n = 0;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      uint32_t b = 0;
#pragma unroll
      for (int u = 0; u < 32; ++u) {
        const int i = w * 32 + u;
        const float v = i < E ? s_log[i * 128] + s_bias[i] : -INFINITY;   // the key, as in the parts
        b |= (v >= lo ? 1u : 0u) << u;
      }
      msk[w] = b;
      n += __popc(b);
    }
    if (n > kRefineCand || (o.gate == 0 && !o.renorm)) {
      cand[0] = -2;
      n = 1;
    } else {
      n = 0;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        for (uint32_t b = msk[w]; b != 0u; b &= b - 1u) cand[n++] = w * 32 + __ffs(b) - 1;
      }
    }
    for (int c = n; c < kRefineCand; ++c) cand[c] = -1;
    return;
  }
  float m = m_part[0];
#pragma unroll
  for (int p = 1; p < NP; ++p) m = fmaxf(m, m_part[p * 128]);
  // The softmax denominator is needed only without renormalisation: with
  // it, the weights exp(l_j - m) / sum over the picks are the renormalised
  // probabilities (the 1e-9 guard then scales with the denominator).
  float S = 1.0f;
  if (o.gate == 0 && !o.renorm) {
    float sp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
    for (int i = 0; i < E; i += 4) {
#pragma unroll
      for (int q = 0; q < 4; ++q)
        sp[q] += i + q < E ? expf(s_log[(i + q) * 128] - m) : 0.f;
    }
    S = (sp[0] + sp[1]) + (sp[2] + sp[3]);
  }
  float sc[KMAX_FUSED];
  float ssum = 0.f;
#pragma unroll
  for (int j = 0; j < KMAX_FUSED; ++j) {
    sc[j] = 0.f;
    if (j < o.k) {
      const float l = s_log[(sid[j] < E ? sid[j] : 0) * 128];   // a pick is an id < E unless keys are NaN
      sc[j] = o.gate == 1 ? 1.0f / (1.0f + expf(-l)) : expf(l - m) / S;
      ssum += sc[j];
    }
  }
  int32_t* irow = o.topk_idx + static_cast<size_t>(t) * o.k;
  float* wrow = o.topk_w + static_cast<size_t>(t) * o.k;
#pragma unroll
  for (int j = 0; j < KMAX_FUSED; ++j) {
    if (j < o.k) {
      irow[j] = sid[j];
      wrow[j] = o.renorm ? sc[j] / (ssum + 1e-9f) : sc[j];
    }
  }
}

template <int NPAD, bool FUSED>
__global__ void __launch_bounds__(RCfg<NPAD, FUSED>::THREADS, 1)
router_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                 int T, int K, int E, const RouterOut out) {
  using C = RCfg<NPAD, FUSED>;
  constexpr uint32_t IDESC = idesc_bf16_f32(RBM, NPAD);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::STAGES * R_A_BYTES;
  float* s_logits = reinterpret_cast<float*>(smem + C::STAGES * C::STAGE_BYTES);
  // fused select: part p's ranking of row r, entry j at [p * PSTRIDE + j * 128 + r]
  constexpr int PSTRIDE = PICKS * 128;
  float* s_pv = reinterpret_cast<float*>(smem + C::STAGES * C::STAGE_BYTES + C::LOGIT_BYTES);
  int* s_pi = reinterpret_cast<int*>(s_pv + C::EPI_WG * PSTRIDE * (FUSED ? 1 : 0));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES +
                                               C::LOGIT_BYTES + C::PICK_BYTES);
  uint64_t* full_bar = bars;
  uint64_t* empty_bar = bars + C::STAGES;
  uint64_t* sfull_bar = bars + 2 * C::STAGES;
  uint64_t* sempty_bar = bars + 2 * C::STAGES + C::NSLOT;
  uint64_t* drain_bar = bars + 2 * C::STAGES + 2 * C::NSLOT;
  // fused select in parts: the other warpgroups' rankings are ready (xfull),
  // the first has merged them and they may be overwritten (xfree)
  uint64_t* xfull_bar = drain_bar + 1;
  uint64_t* xfree_bar = drain_bar + 2;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ __align__(16) float s_off[NPAD];
  __shared__ __align__(16) float s_bias[NPAD];
  __shared__ float s_mpart[FUSED ? C::EPI_WG * 128 : 1];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles = (T + RBM - 1) / RBM;
  const int kblocks = K / RBK;
  const int chunks = (kblocks + KCH - 1) / KCH;

  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int s = 0; s < C::NSLOT; ++s) {
      mbar_init(&sfull_bar[s], 1);
      mbar_init(&sempty_bar[s], 4 * C::EPI_WG);
    }
    mbar_init(drain_bar, 1);
    mbar_init(xfull_bar, 128 * (C::EPI_WG > 1 ? C::EPI_WG - 1 : 1));
    mbar_init(xfree_bar, 128);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(&s_tmem, C::TMEM_COLS);
    tmem_relinquish();
  }
  pdl_wait();   // everything above touches no global memory
  if (FUSED && warp >= 2) {
    for (int e = threadIdx.x - 64; e < NPAD; e += 128) {
      s_off[e] = (e < E && out.offset) ? out.offset[e] : 0.f;
      s_bias[e] = (e < E && out.bias) ? out.bias[e] : 0.f;
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
      const uint64_t keep_x = l2_evict_last_policy();
      for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&full_bar[stage], C::STAGE_BYTES);
          tma_load_2d_hint(sA + stage * R_A_BYTES, &tmX, &full_bar[stage], kb * RBK, tile * RBM,
                           keep_x);
          tma_load_2d(sB + stage * C::B_BYTES, &tmW, &full_bar[stage], kb * RBK, 0);
          issued_mask |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      pdl_trigger();   // all loads issued: the next kernel may launch
      if (!ok) {
        for (int s = 0; s < C::STAGES; ++s) {
          if (!(issued_mask & (1u << s))) continue;
          const unsigned long long t0 = globaltimer_ns();
          while (!mbar_try_wait(&full_bar[s], (issued_phase >> s) & 1u))
            if (globaltimer_ns() - t0 > kWaitLimitNs) break;
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0, cc = 0;
      uint32_t phase = 0;
      bool ok = true, issued = false;
      for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
        for (int ch = 0; ch < chunks && ok; ++ch, ++cc) {
          const int slot = cc % C::NSLOT;
          const uint32_t sph = (cc / C::NSLOT) & 1;
          if (!mbar_wait(&sempty_bar[slot], sph ^ 1u, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d = tmem + slot * NPAD;
          const int kb_end = (ch + 1) * KCH < kblocks ? (ch + 1) * KCH : kblocks;
          for (int kb = ch * KCH; kb < kb_end; ++kb) {
            if (!mbar_wait(&full_bar[stage], phase, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint32_t a = smem_u32(sA + stage * R_A_BYTES);
            const uint32_t b = smem_u32(sB + stage * C::B_BYTES);
#pragma unroll
            for (int kk = 0; kk < RBK / 16; ++kk)
              tc_mma_f16(d, smem_desc_sw128(a + kk * 32), smem_desc_sw128(b + kk * 32), IDESC,
                         (kb > ch * KCH || kk > 0) ? 1u : 0u);
            issued = true;
            tc_commit(&empty_bar[stage]);
            if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
          }
          if (!ok) break;
          tc_commit(&sfull_bar[slot]);
        }
      }
      if (!ok && issued) {
        tc_commit(drain_bar);
        const unsigned long long t0 = globaltimer_ns();
        while (!mbar_try_wait(drain_bar, 0))
          if (globaltimer_ns() - t0 > kWaitLimitNs) break;
      }
    }
  } else {
    const int ew = warp - 2;                 // epilogue warp 0 .. 4*EPI_WG-1
    const int wg = ew >> 2;                  // column part of this warpgroup
    const int q = warp & 3;                  // TMEM lane quadrant of this warp
    const int row = q * 32 + lane;
    int cc = 0, it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x, ++it) {
      float acc[C::COLS];
#pragma unroll
      for (int i = 0; i < C::COLS; ++i) acc[i] = 0.f;
      for (int ch = 0; ch < chunks; ++ch, ++cc) {
        const int slot = cc % C::NSLOT;
        const uint32_t sph = (cc / C::NSLOT) & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&sfull_bar[slot], sph, abort_flag));
        if (!ok) break;
        tc_fence_after();
        const uint32_t taddr =
            tmem + slot * NPAD + wg * C::COLS + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll
        for (int c = 0; c < C::COLS / 16; ++c) {
          uint32_t v[16];
          tmem_ld16(taddr + c * 16, v);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) acc[c * 16 + i] += __uint_as_float(v[i]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sempty_bar[slot]);
      }
      if (!ok) break;
      const int t = tile * RBM + row;
      if constexpr (FUSED) {
        // every thread ranks its part of the row (rows past T too, so that
        // all take part in the exchange); the first warpgroup merges
        const int rounds = out.k < E ? out.k + 1 : out.k;
        if (C::EPI_WG > 1 && wg > 0 && it > 0) {
          // the first warpgroup must have merged the previous tile
          ok = __all_sync(0xffffffffu, mbar_wait(xfree_bar, (it - 1) & 1, abort_flag));
          if (!ok) break;
        }
        s_mpart[wg * 128 + row] =
            route_part<C::COLS>(acc, s_logits + row, s_off, s_bias, wg * C::COLS, E, rounds,
                                s_pv + wg * PSTRIDE + row, s_pi + wg * PSTRIDE + row);
        if (C::EPI_WG > 1) {
          if (wg > 0) {
            mbar_arrive(xfull_bar);
            continue;
          }
          ok = __all_sync(0xffffffffu, mbar_wait(xfull_bar, it & 1, abort_flag));
          if (!ok) break;
        }
        if (t < T)
          route_finish<C::EPI_WG>(s_pv + row, s_pi + row, PSTRIDE, s_mpart + row,
                                  s_logits + row, s_bias, E, t, out);
        if (C::EPI_WG > 1) mbar_arrive(xfree_bar);
      } else {
        if (t >= T) continue;
        float* dst = out.logits + static_cast<size_t>(t) * E + wg * C::COLS;
        const int ncol = E - wg * C::COLS;
        if ((E & 3) == 0 && ncol >= C::COLS) {
#pragma unroll
          for (int i = 0; i < C::COLS; i += 4)
            *reinterpret_cast<float4*>(dst + i) =
                make_float4(acc[i], acc[i + 1], acc[i + 2], acc[i + 3]);
        } else {
#pragma unroll
          for (int i = 0; i < C::COLS; ++i)
            if (i < ncol) dst[i] = acc[i];
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && s_abort) atomicOr(out.status, kDevTimeout);
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// Looked up once per process; the initialisation of a function-local
// static is thread-safe.
EncodeTiledFn encode_fn() {
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

bool map2d(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(RBK), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

template <int NPAD, bool FUSED>
cudaError_t launch_router(const CUtensorMap& mx, const CUtensorMap& mw, int T, int K, int E,
                          const RouterOut& out, cudaStream_t stream) {
  using C = RCfg<NPAD, FUSED>;
  auto kern = router_tc_kernel<NPAD, FUSED>;
  static std::atomic<unsigned long long> attr_done{0};
  int dev = 0;
  cudaGetDevice(&dev);
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(attr_done.load(std::memory_order_acquire) & bit)) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_done.fetch_or(bit, std::memory_order_acq_rel);
  }
  int sms = 0;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int tiles = (T + RBM - 1) / RBM;
  const int grid = tiles < sms ? tiles : (sms > 0 ? sms : 148);
  return launch_pdl(kern, dim3(grid), dim3(C::THREADS), C::SMEM_BYTES, stream, mx, mw, T, K, E,
                    out);
}

int npad_for(int E) {
  int npad = 16;
  while (npad < E) npad *= 2;
  return npad;
}

bool maps(const void* x, int T, const void* w_router, int E, int K, CUtensorMap* mx,
          CUtensorMap* mw) {
  return map2d(mx, x, T, K, RBM) && map2d(mw, w_router, E, K, npad_for(E));
}

}  // namespace

bool router_fused_supported(int E, int k) { return npad_for(E) <= 128 && k <= KMAX_FUSED; }

cudaError_t router_logits_tc(const void* x, int T, const void* w_router, int E, int K,
                             float* logits, uint32_t* status, cudaStream_t stream) {
  if (T <= 0) return cudaSuccess;
  const int npad = npad_for(E);
  if (npad > 256) return cudaErrorInvalidValue;
  CUtensorMap mx, mw;
  if (!maps(x, T, w_router, E, K, &mx, &mw)) return cudaErrorInvalidValue;
  RouterOut o{logits, nullptr, nullptr, 0, 0, 0, nullptr, nullptr, nullptr, nullptr, nullptr,
              status};
  switch (npad) {
    case 16: return launch_router<16, false>(mx, mw, T, K, E, o, stream);
    case 32: return launch_router<32, false>(mx, mw, T, K, E, o, stream);
    case 64: return launch_router<64, false>(mx, mw, T, K, E, o, stream);
    case 128: return launch_router<128, false>(mx, mw, T, K, E, o, stream);
    default: return launch_router<256, false>(mx, mw, T, K, E, o, stream);
  }
}

cudaError_t router_topk_tc(const void* x, int T, const void* w_router, int E, int K,
                           const float* logit_offset, const float* sel_bias, int k, int gate,
                           int renorm, int32_t* topk_idx, float* topk_w, int32_t* refine_count,
                           int32_t* refine_list, int32_t* refine_cand, uint32_t* status,
                           cudaStream_t stream) {
  if (T <= 0) return cudaSuccess;
  if (!router_fused_supported(E, k)) return cudaErrorInvalidValue;
  CUtensorMap mx, mw;
  if (!maps(x, T, w_router, E, K, &mx, &mw)) return cudaErrorInvalidValue;
  RouterOut o{nullptr, logit_offset, sel_bias, k, gate, renorm, topk_idx, topk_w,
              refine_count, refine_list, refine_cand, status};
  switch (npad_for(E)) {
    case 16: return launch_router<16, true>(mx, mw, T, K, E, o, stream);
    case 32: return launch_router<32, true>(mx, mw, T, K, E, o, stream);
    case 64: return launch_router<64, true>(mx, mw, T, K, E, o, stream);
    default: return launch_router<128, true>(mx, mw, T, K, E, o, stream);
  }
}

}  // namespace moe
