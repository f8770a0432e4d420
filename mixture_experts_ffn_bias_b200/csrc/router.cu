// Router: logits, gate, biased selection, top-k and combine weights.
//
// Follows SigmoidRouter.forward of the "moe-200m-qwen3-100b" README (fp32
// linear with autocast off, sigmoid scores, selection logits = logits + bias,
// top-k of the selection logits, weights gathered from the unbiased scores and
// divided by their sum + 1e-9) and the qwen3 preset of SpecForge PR #930
// (softmax over all experts, top-k weights renormalised).
//
// Precision: x and w_router hold bf16 (or fp32) values.  Products are formed
// in fp32 (exact for bf16 x bf16), summed in fp32 over 32-wide K chunks and the
// chunk sums are added in fp64, so a logit is within ~1e-8 of the exact dot
// product for the layer sizes used here.  Selection keys, gate scores and the
// renormalisation are then evaluated in fp64 and the weights stored as fp32.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.h"

namespace moe {
namespace {

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

constexpr int RT_TOK = 64;    // tokens per block
constexpr int RT_EXP = 32;    // experts per block
constexpr int RT_KC = 32;     // K chunk accumulated in fp32

template <typename Tin>
__global__ void __launch_bounds__(256)
router_logits_kernel(const Tin* __restrict__ x, const Tin* __restrict__ wr,
                     const float* __restrict__ offset, int T, int d, int E,
                     double* __restrict__ logits) {
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

constexpr int kMaxPerLane = 8;   // E <= 256 = 8 x 32

// One warp per token.  Lane l holds experts l, l+32, ...
__global__ void __launch_bounds__(256)
router_select_kernel(const double* __restrict__ logits, const float* __restrict__ bias, int T,
                     int E, int k, int gate, int renorm, int32_t* __restrict__ topk_idx,
                     float* __restrict__ topk_w) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  double l[kMaxPerLane], key[kMaxPerLane], s[kMaxPerLane];
  bool taken[kMaxPerLane];
  double lmax = -INFINITY;
#pragma unroll
  for (int i = 0; i < kMaxPerLane; ++i) {
    const int e = lane + 32 * i;
    if (e < E) {
      l[i] = logits[static_cast<size_t>(t) * E + e];
      key[i] = l[i] + (bias ? static_cast<double>(bias[e]) : 0.0);
      taken[i] = false;
      lmax = fmax(lmax, l[i]);
    } else {
      l[i] = -INFINITY;
      key[i] = -INFINITY;
      taken[i] = true;
    }
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
    topk_idx[static_cast<size_t>(t) * k + lane] = my_idx;
    topk_w[static_cast<size_t>(t) * k + lane] = static_cast<float>(my_w);
  }
}

}  // namespace

cudaError_t router_logits(bool bf16, const void* x, const void* w_router,
                          const float* logit_offset, int T, int d, int E, double* logits,
                          cudaStream_t stream) {
  dim3 grid((T + RT_TOK - 1) / RT_TOK, (E + RT_EXP - 1) / RT_EXP);
  if (bf16)
    router_logits_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(w_router),
        logit_offset, T, d, E, logits);
  else
    router_logits_kernel<float><<<grid, 256, 0, stream>>>(
        static_cast<const float*>(x), static_cast<const float*>(w_router), logit_offset, T, d, E,
        logits);
  return cudaGetLastError();
}

cudaError_t router_select(const double* logits, const float* sel_bias, int T, int E, int k,
                          int gate, int renorm, int32_t* topk_idx, float* topk_w,
                          cudaStream_t stream) {
  const int warps = 8;
  router_select_kernel<<<(T + warps - 1) / warps, warps * 32, 0, stream>>>(
      logits, sel_bias, T, E, k, gate, renorm, topk_idx, topk_w);
  return cudaGetLastError();
}

}  // namespace moe
