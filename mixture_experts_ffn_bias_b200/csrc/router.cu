// Router: logits, gate, biased selection, top-k and combine weights.
//
// Follows SigmoidRouter.forward of the "moe-200m-qwen3-100b" README (fp32
// linear with autocast off, sigmoid scores, selection logits = logits + bias,
// top-k of the selection logits, weights gathered from the unbiased scores and
// divided by their sum + 1e-9) and the qwen3 preset of SpecForge PR #930
// (softmax over all experts, top-k weights renormalised).
//
// bf16 layers (the production path):
//   1. logits = x . Wr^T on the tensor cores (router_sm100.cu): exact bf16 x
//      bf16 products, fp32 accumulation in 128-wide K chunks.  With E <= 128
//      and k <= 8 the same kernel also selects (fused select) and lists the
//      near-tie tokens with their candidate experts; otherwise it writes the
//      logits and
//   2. router_select_fast_kernel decides: one warp per token, fp32 keys and
//      gate; a token whose k-th / (k+1)-th keys, or two adjacent keys inside
//      its top-k, are closer than kRefineMargin is not decided here but
//      appended to a refine list.
//   3. router_refine_kernel: for each listed token, exact logits (fp64 sums of
//      exact products) over its candidates (or all experts) and the
//      selection in fp64.
//   The fp32 accumulation error of a logit (< 5e-6) is far below the margin,
//   so every token's decision equals the one taken on exact logits.
// fp32 layers: logits on CUDA cores (fp32 products summed in fp32 over
// 32-wide K chunks, chunk sums added in fp64), selection in fp64.
//
// Key variants (KeyOpts, moe_router_topk_opts): the bias added to the gate
// score instead of the logit (the score-space placement of the "noaux_tc"
// balance bias named on the page-3 model card), and a caller-drawn selection
// noise [T, E] added to every key (the training-time exploration noise of
// SigmoidRouter.forward).  Every select path forms the same keys; the
// variants run the unfused bf16 path with re-decision over all experts.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.h"
#include "launch.cuh"
#include "router_exact.cuh"

namespace moe {
namespace {

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

constexpr int RT_TOK = 64;    // tokens per block
constexpr int RT_EXP = 32;    // experts per block
constexpr int RT_KC = 32;     // K chunk accumulated in fp32

// ---------------------------------------------------------------- fp32 layers
template <typename Tin>
__global__ void __launch_bounds__(256)
router_logits_kernel(const Tin* __restrict__ x, const Tin* __restrict__ wr,
                     const float* __restrict__ offset, int T, int d, int E,
                     double* __restrict__ logits) {
  pdl_trigger();
  pdl_wait();
  __shared__ float xs[RT_KC][RT_TOK + 4];
  __shared__ float ws[RT_KC][RT_EXP + 4];
  const int tid = threadIdx.x;
  const int tx = tid & 7;    // experts 4*tx .. 4*tx+3 of the block
  const int ty = tid >> 3;   // tokens 2*ty, 2*ty+1 of the block
  const int t0 = blockIdx.x * RT_TOK;
  const int e0 = blockIdx.y * RT_EXP;
  double dacc[2][4];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) dacc[i][j] = 0.0;

  for (int k0 = 0; k0 < d; k0 += RT_KC) {
    {
      const int tt = tid >> 2, kk = (tid & 3) * 8, t = t0 + tt;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int c = k0 + kk + i;
        xs[kk + i][tt] = (t < T && c < d) ? to_f32(x[static_cast<size_t>(t) * d + c]) : 0.0f;
      }
    }
    {
      const int ee = tid >> 3, kk = (tid & 7) * 4, e = e0 + ee;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int c = k0 + kk + i;
        ws[kk + i][ee] = (e < E && c < d) ? to_f32(wr[static_cast<size_t>(e) * d + c]) : 0.0f;
      }
    }
    __syncthreads();
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll 8
    for (int kk = 0; kk < RT_KC; ++kk) {
      const float a0 = xs[kk][2 * ty], a1 = xs[kk][2 * ty + 1];
      const float4 b = *reinterpret_cast<const float4*>(&ws[kk][4 * tx]);
      acc[0][0] = fmaf(a0, b.x, acc[0][0]);
      acc[0][1] = fmaf(a0, b.y, acc[0][1]);
      acc[0][2] = fmaf(a0, b.z, acc[0][2]);
      acc[0][3] = fmaf(a0, b.w, acc[0][3]);
      acc[1][0] = fmaf(a1, b.x, acc[1][0]);
      acc[1][1] = fmaf(a1, b.y, acc[1][1]);
      acc[1][2] = fmaf(a1, b.z, acc[1][2]);
      acc[1][3] = fmaf(a1, b.w, acc[1][3]);
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) dacc[i][j] += static_cast<double>(acc[i][j]);
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int t = t0 + 2 * ty + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = e0 + 4 * tx + j;
      if (e < E)
        logits[static_cast<size_t>(t) * E + e] =
            dacc[i][j] + (offset ? static_cast<double>(offset[e]) : 0.0);
    }
  }
}

// Selection, gate and weights for one token in fp64, done by one warp.  `l`
// holds the logits of experts lane + 32 i (offset already added); keys are
// (space ? score : logit) + bias (+ noise_row[e]).
__device__ void warp_select_fp64(const double (&l)[kMaxPerLane], const float* __restrict__ bias,
                                 int E, int k, int gate, int renorm, int space,
                                 const float* __restrict__ noise_row,
                                 int32_t* __restrict__ idx_row, float* __restrict__ w_row) {
  const int lane = threadIdx.x & 31;
  double key[kMaxPerLane], s[kMaxPerLane];
  bool taken[kMaxPerLane];
  double lmax = -INFINITY;
#pragma unroll
  for (int i = 0; i < kMaxPerLane; ++i) {
    const int e = lane + 32 * i;
    taken[i] = e >= E;
    if (e < E) lmax = fmax(lmax, l[i]);
  }
  if (gate == 1) {  // sigmoid
#pragma unroll
    for (int i = 0; i < kMaxPerLane; ++i) s[i] = 1.0 / (1.0 + exp(-l[i]));
  } else {          // softmax over all E experts, max subtracted
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lmax = fmax(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
    double sum = 0.0;
#pragma unroll
    for (int i = 0; i < kMaxPerLane; ++i) {
      s[i] = (lane + 32 * i < E) ? exp(l[i] - lmax) : 0.0;
      sum += s[i];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
#pragma unroll
    for (int i = 0; i < kMaxPerLane; ++i) s[i] = s[i] / sum;
  }
#pragma unroll
  for (int i = 0; i < kMaxPerLane; ++i) {
    const int e = lane + 32 * i;
    key[i] = e < E ? (space ? s[i] : l[i]) + (bias ? static_cast<double>(bias[e]) : 0.0) +
                         (noise_row ? static_cast<double>(noise_row[e]) : 0.0)
                   : -INFINITY;
  }
  int my_idx = 0;
  double my_w = 0.0, wsum = 0.0;
  for (int j = 0; j < k; ++j) {
    double bk = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < kMaxPerLane; ++i) {
      const int e = lane + 32 * i;
      if (!taken[i] && (key[i] > bk || (key[i] == bk && e < be))) {
        bk = key[i];
        be = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const double ok = __shfl_xor_sync(0xffffffffu, bk, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (ok > bk || (ok == bk && oe < be)) {
        bk = ok;
        be = oe;
      }
    }
    const int owner = be & 31, slot = be >> 5;
    double sc = 0.0;
#pragma unroll
    for (int i = 0; i < kMaxPerLane; ++i) {
      if (lane == owner && i == slot) {
        taken[i] = true;
        sc = s[i];
      }
    }
    sc = __shfl_sync(0xffffffffu, sc, owner);
    if (lane == j) {
      my_idx = be;
      my_w = sc;
    }
    wsum += sc;
  }
  if (renorm) my_w = my_w / (wsum + 1e-9);
  if (lane < k) {
    idx_row[lane] = my_idx;
    w_row[lane] = static_cast<float>(my_w);
  }
}

// One warp per token, fp64 logits.
__global__ void __launch_bounds__(256)
router_select_kernel(const double* __restrict__ logits, const float* __restrict__ bias, int T,
                     int E, int k, int gate, int renorm, int space,
                     const float* __restrict__ noise, int32_t* __restrict__ topk_idx,
                     float* __restrict__ topk_w) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  double l[kMaxPerLane];
#pragma unroll
  for (int i = 0; i < kMaxPerLane; ++i) {
    const int e = lane + 32 * i;
    l[i] = e < E ? logits[static_cast<size_t>(t) * E + e] : -INFINITY;
  }
  warp_select_fp64(l, bias, E, k, gate, renorm, space,
                   noise ? noise + static_cast<size_t>(t) * E : nullptr,
                   topk_idx + static_cast<size_t>(t) * k, topk_w + static_cast<size_t>(t) * k);
}

// ---------------------------------------------------------------- bf16 layers
// One warp per token, fp32 logits from the tensor cores.
__global__ void __launch_bounds__(256)
router_select_fast_kernel(const float* __restrict__ logits, const float* __restrict__ offset,
                          const float* __restrict__ bias, int T, int E, int k, int gate,
                          int renorm, int space, const float* __restrict__ noise,
                          int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
                          int32_t* __restrict__ refine_count,
                          int32_t* __restrict__ refine_list) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  float l[kMaxPerLane], key[kMaxPerLane];
  bool taken[kMaxPerLane];
  float lmax = -INFINITY;
#pragma unroll
  for (int i = 0; i < kMaxPerLane; ++i) {
    const int e = lane + 32 * i;
    if (e < E) {
      l[i] = logits[static_cast<size_t>(t) * E + e] + (offset ? offset[e] : 0.0f);
      key[i] = l[i];
      taken[i] = false;
      lmax = fmaxf(lmax, l[i]);
    } else {
      l[i] = -INFINITY;
      key[i] = -INFINITY;
      taken[i] = true;
    }
  }
  // Score-space softmax keys are probabilities: their error scales with the
  // largest one (1 / sum), so the re-decision margin does too, with a floor
  // for the rounding of the bias addition.
  float margin = kRefineMargin;
  if (space) {   // key base = the gate score
    if (gate == 1) {
#pragma unroll
      for (int i = 0; i < kMaxPerLane; ++i) key[i] = 1.0f / (1.0f + expf(-l[i]));
    } else {
      float mm = lmax;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mm = fmaxf(mm, __shfl_xor_sync(0xffffffffu, mm, o));
      float sum = 0.f;
#pragma unroll
      for (int i = 0; i < kMaxPerLane; ++i) {
        key[i] = expf(l[i] - mm);   // 0 past E
        sum += key[i];
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
#pragma unroll
      for (int i = 0; i < kMaxPerLane; ++i) key[i] = key[i] / sum;
      margin = fmaxf(kRefineMargin / sum, 1e-5f);
    }
  }
#pragma unroll
  for (int i = 0; i < kMaxPerLane; ++i) {
    const int e = lane + 32 * i;
    if (e < E)
      key[i] += (bias ? bias[e] : 0.0f) + (noise ? noise[static_cast<size_t>(t) * E + e] : 0.0f);
    else
      key[i] = -INFINITY;
  }
  // top-(k+1) keys, descending, ties -> lower expert id
  const int rounds = k < E ? k + 1 : k;
  float prev = 0.f, min_gap = INFINITY, edge_gap = INFINITY;
  int my_idx = 0;
  float my_l = 0.f;
  for (int j = 0; j < rounds; ++j) {
    float bk = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < kMaxPerLane; ++i) {
      const int e = lane + 32 * i;
      if (!taken[i] && (key[i] > bk || (key[i] == bk && e < be))) {
        bk = key[i];
        be = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ok = __shfl_xor_sync(0xffffffffu, bk, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (ok > bk || (ok == bk && oe < be)) {
        bk = ok;
        be = oe;
      }
    }
    const int owner = be & 31, slot = be >> 5;
    float lsel = 0.f;
#pragma unroll
    for (int i = 0; i < kMaxPerLane; ++i) {
      if (lane == owner && i == slot) {
        taken[i] = true;
        lsel = l[i];
      }
    }
    lsel = __shfl_sync(0xffffffffu, lsel, owner);
    if (j > 0) {
      const float gap = prev - bk;
      if (j < k) min_gap = fminf(min_gap, gap);
      else edge_gap = gap;
    }
    prev = bk;
    if (lane == j && j < k) {
      my_idx = be;
      my_l = lsel;
    }
  }
  if (fminf(min_gap, edge_gap) < margin) {
    if (lane == 0) refine_list[atomicAdd(refine_count, 1)] = t;
    return;
  }
  // gate scores of the chosen experts and the weights
  float s;
  if (gate == 1) {
    s = 1.0f / (1.0f + expf(-my_l));
  } else {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lmax = fmaxf(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < kMaxPerLane; ++i)
      if (lane + 32 * i < E) sum += expf(l[i] - lmax);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    s = expf(my_l - lmax) / sum;
  }
  float ssum = lane < k ? s : 0.f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ssum += __shfl_xor_sync(0xffffffffu, ssum, o);
  if (renorm) s = s / (ssum + 1e-9f);
  if (lane < k) {
    topk_idx[static_cast<size_t>(t) * k + lane] = my_idx;
    topk_w[static_cast<size_t>(t) * k + lane] = s;
  }
}

// Exact re-decision of listed tokens: one block per listed token.  The
// chain of dependent memory accesses is kept short: the list length, then the
// token and its candidate experts together, then the x row and the router
// rows together (every warp loads the token's x row into registers and each
// of its candidates' rows in full before it multiplies), then the decision
// (refine_select of router_exact.cuh) by warp 0.
__global__ void __launch_bounds__(256)
router_refine_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ wr,
                     const float* __restrict__ offset, const float* __restrict__ bias, int d,
                     int E, int k, int gate, int renorm, int space,
                     const float* __restrict__ noise, const int32_t* __restrict__ refine_count,
                     const int32_t* __restrict__ refine_list,
                     const int32_t* __restrict__ refine_cand, int32_t* __restrict__ topk_idx,
                     float* __restrict__ topk_w) {
  pdl_trigger();
  pdl_wait();
  constexpr int kVecs = 8;                  // 16-byte pieces of a row per lane held at once
  __shared__ double s_l[256];
  __shared__ int s_e[256];
  __shared__ int s_n, s_t, s_all;
  const int n_list = *refine_count;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nv = d / 8;                     // 16-byte pieces of a row
  for (int i = blockIdx.x; i < n_list; i += gridDim.x) {
    if (warp == 0) {
      // the token and its candidates (a prefix of the list row, -1 after it;
      // -2 first: all experts) are read together
      const int t = refine_list[i];
      int ce = -1;
      if (refine_cand && lane < kRefineCand) ce = refine_cand[static_cast<size_t>(i) * kRefineCand + lane];
      const bool all = refine_cand == nullptr || __shfl_sync(0xffffffffu, ce, 0) == -2;
      const int n = all ? E : __popc(__ballot_sync(0xffffffffu, ce >= 0));
      if (!all && lane < kRefineCand) s_e[lane] = ce;
      if (lane == 0) {
        s_n = n;
        s_t = t;
        s_all = all ? 1 : 0;
      }
    }
    __syncthreads();
    const int n = s_n, t = s_t;
    const bool all = s_all != 0;
    const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * d);
    for (int c = warp; c < n; c += 8) {
      const int e = all ? c : s_e[c];
      const uint4* wrow = reinterpret_cast<const uint4*>(wr + static_cast<size_t>(e) * d);
      double a[4] = {0.0, 0.0, 0.0, 0.0};
      for (int v0 = lane; v0 < nv; v0 += 32 * kVecs) {
        uint4 ux[kVecs], uw[kVecs];
#pragma unroll
        for (int u = 0; u < kVecs; ++u) {
          const int v = v0 + 32 * u;
          ux[u] = v < nv ? __ldg(xr + v) : make_uint4(0u, 0u, 0u, 0u);
          uw[u] = v < nv ? __ldg(wrow + v) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < kVecs; ++u) {
          const __nv_bfloat16* hx = reinterpret_cast<const __nv_bfloat16*>(&ux[u]);
          const __nv_bfloat16* hw = reinterpret_cast<const __nv_bfloat16*>(&uw[u]);
#pragma unroll
          for (int j = 0; j < 8; ++j)   // bf16 x bf16 products are exact in fp32; fp64 sums
            a[j & 3] += static_cast<double>(__bfloat162float(hw[j]) * __bfloat162float(hx[j]));
        }
      }
      double sum = (a[0] + a[1]) + (a[2] + a[3]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (lane == 0) {
        s_l[c] = sum + (offset ? static_cast<double>(offset[e]) : 0.0);
        if (all) s_e[c] = c;
      }
    }
    __syncthreads();
    if (warp == 0)
      refine_select(s_l, s_e, n, bias, k, gate, renorm, all, space,
                    noise ? noise + static_cast<size_t>(t) * E : nullptr,
                    topk_idx + static_cast<size_t>(t) * k, topk_w + static_cast<size_t>(t) * k);
    __syncthreads();
  }
}

__global__ void add_row_offset_kernel(float* __restrict__ logits, const float* __restrict__ off,
                                      long long n, int E) {
  pdl_trigger();
  pdl_wait();
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x)
    logits[i] += off[i % E];
}

}  // namespace

cudaError_t add_row_offset(float* logits, const float* offset, int T, int E, cudaStream_t stream) {
  const long long n = static_cast<long long>(T) * E;
  const int grid = static_cast<int>((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
  return launch_pdl(add_row_offset_kernel, dim3(grid), dim3(256), 0, stream, logits, offset, n, E);
}

cudaError_t router_logits(bool bf16, const void* x, const void* w_router,
                          const float* logit_offset, int T, int d, int E, double* logits,
                          cudaStream_t stream) {
  dim3 grid((T + RT_TOK - 1) / RT_TOK, (E + RT_EXP - 1) / RT_EXP);
  if (bf16)
    return launch_pdl(router_logits_kernel<__nv_bfloat16>, grid, dim3(256), 0, stream,
                      static_cast<const __nv_bfloat16*>(x),
                      static_cast<const __nv_bfloat16*>(w_router), logit_offset, T, d, E,
                      logits);
  return launch_pdl(router_logits_kernel<float>, grid, dim3(256), 0, stream,
                    static_cast<const float*>(x), static_cast<const float*>(w_router),
                    logit_offset, T, d, E, logits);
}

cudaError_t router_select(const double* logits, const float* sel_bias, int T, int E, int k,
                          int gate, int renorm, const KeyOpts& ko, int32_t* topk_idx,
                          float* topk_w, cudaStream_t stream) {
  const int warps = 8;
  return launch_pdl(router_select_kernel, dim3((T + warps - 1) / warps), dim3(warps * 32), 0,
                    stream, logits, sel_bias, T, E, k, gate, renorm, ko.space, ko.noise, topk_idx,
                    topk_w);
}

cudaError_t router_select_fast(const float* logits, const float* logit_offset,
                               const float* sel_bias, int T, int E, int k, int gate, int renorm,
                               const KeyOpts& ko, int32_t* topk_idx, float* topk_w,
                               int32_t* refine_count, int32_t* refine_list, cudaStream_t stream) {
  const int warps = 8;
  return launch_pdl(router_select_fast_kernel, dim3((T + warps - 1) / warps), dim3(warps * 32), 0,
                    stream, logits, logit_offset, sel_bias, T, E, k, gate, renorm, ko.space,
                    ko.noise, topk_idx, topk_w, refine_count, refine_list);
}

cudaError_t router_refine(const void* x, const void* w_router, const float* logit_offset,
                          const float* sel_bias, int T, int d, int E, int k, int gate,
                          int renorm, const KeyOpts& ko, const int32_t* refine_count,
                          const int32_t* refine_list, const int32_t* refine_cand,
                          int32_t* topk_idx, float* topk_w, int sms, cudaStream_t stream) {
  int grid = 2 * sms;
  if (grid > T) grid = T;
  if (grid < 1) grid = 1;
  return launch_pdl(router_refine_kernel, dim3(grid), dim3(256), 0, stream,
                    static_cast<const __nv_bfloat16*>(x),
                    static_cast<const __nv_bfloat16*>(w_router), logit_offset, sel_bias, d, E, k,
                    gate, renorm, ko.space, ko.noise, refine_count, refine_list, refine_cand,
                    topk_idx, topk_w);
}

}  // namespace moe
