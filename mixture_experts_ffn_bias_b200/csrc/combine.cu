// Weighted un-permute / combine and the selection-bias controller update.
//
// combine:  out[t] = y_shared[t] + sum_{j<k} w[t, j] * y_perm[slot_pos[t, j]]
// ("moe-200m-qwen3-100b" README, "Architecture diagram": routed experts and
// the always-on shared expert, then the weighted sum).  One warp per token,
// 16-byte vector loads of the k expert rows, fp32 accumulation in j order,
// one store of the output row.
//
// bias update: step_bias_update of the same README ("SigmoidRouter"), one
// correctly rounded fp32 operation per step, no fused multiply-add.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.h"
#include "launch.cuh"

namespace moe {
namespace {

template <bool BF16>
struct Vec;
template <>
struct Vec<true> {
  static constexpr int N = 8;
  __device__ static void load(const uint4& v, float* f) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 p = __bfloat1622float2(h[i]);
      f[2 * i] = p.x;
      f[2 * i + 1] = p.y;
    }
  }
  __device__ static uint4 store(const float* f) {
    uint4 v;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    return v;
  }
};
template <>
struct Vec<false> {
  static constexpr int N = 4;
  __device__ static void load(const uint4& v, float* f) {
    f[0] = __uint_as_float(v.x);
    f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z);
    f[3] = __uint_as_float(v.w);
  }
  __device__ static uint4 store(const float* f) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                      __float_as_uint(f[3]));
  }
};

// KT > 0: k == KT known at compile time, so each lane issues the loads of all
// k rows (and the shared row) before it accumulates; KT == 0: any k.  A slot
// outside [0, T*k) (a skipped pair, or a caller's bad slot) contributes
// nothing.
template <bool BF16, int KT>
__global__ void __launch_bounds__(256)
combine_kernel(const uint4* __restrict__ y_perm, const int32_t* __restrict__ slot_pos,
               const float* __restrict__ topk_w, const uint4* __restrict__ y_shared,
               uint4* __restrict__ out, int T, int vecs, int k_rt) {
  pdl_trigger();
  pdl_wait();
  using V = Vec<BF16>;
  const int k = KT > 0 ? KT : k_rt;
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  int my_slot = -1;
  float my_w = 0.f;
  if (lane < k) {
    my_slot = slot_pos[static_cast<size_t>(t) * k + lane];
    my_w = topk_w[static_cast<size_t>(t) * k + lane];
    if (static_cast<long long>(my_slot) >= static_cast<long long>(T) * k) my_slot = -1;
  }
  if constexpr (KT > 0) {
    int sl[KT > 0 ? KT : 1];
    float wj[KT > 0 ? KT : 1];
#pragma unroll
    for (int j = 0; j < KT; ++j) {
      sl[j] = __shfl_sync(0xffffffffu, my_slot, j);
      wj[j] = __shfl_sync(0xffffffffu, my_w, j);
    }
    for (int c = lane; c < vecs; c += 32) {
      uint4 v[KT > 0 ? KT : 1];
      uint4 vs = make_uint4(0u, 0u, 0u, 0u);
      if (y_shared) vs = __ldcs(y_shared + static_cast<size_t>(t) * vecs + c);
#pragma unroll
      for (int j = 0; j < KT; ++j)
        v[j] = sl[j] >= 0 ? __ldcs(y_perm + static_cast<size_t>(sl[j]) * vecs + c)
                          : make_uint4(0u, 0u, 0u, 0u);
      float acc[V::N];
      if (y_shared) {
        V::load(vs, acc);
      } else {
#pragma unroll
        for (int i = 0; i < V::N; ++i) acc[i] = 0.f;
      }
#pragma unroll
      for (int j = 0; j < KT; ++j) {
        float f[V::N];
        V::load(v[j], f);
#pragma unroll
        for (int i = 0; i < V::N; ++i) acc[i] = fmaf(wj[j], f[i], acc[i]);
      }
      out[static_cast<size_t>(t) * vecs + c] = V::store(acc);
    }
  } else {
    for (int c = lane; c < vecs; c += 32) {
      float acc[V::N];
      if (y_shared) {
        V::load(__ldg(y_shared + static_cast<size_t>(t) * vecs + c), acc);
      } else {
#pragma unroll
        for (int i = 0; i < V::N; ++i) acc[i] = 0.f;
      }
      for (int j = 0; j < k; ++j) {
        const int s = __shfl_sync(0xffffffffu, my_slot, j);
        const float w = __shfl_sync(0xffffffffu, my_w, j);
        if (s < 0) continue;
        float f[V::N];
        V::load(__ldg(y_perm + static_cast<size_t>(s) * vecs + c), f);
#pragma unroll
        for (int i = 0; i < V::N; ++i) acc[i] = fmaf(w, f[i], acc[i]);
      }
      out[static_cast<size_t>(t) * vecs + c] = V::store(acc);
    }
  }
}

__global__ void __launch_bounds__(256)
bias_update_kernel(const int32_t* __restrict__ counts, float* __restrict__ bias, int E,
                   float target, float thresh, float starved_add, float rate, float clampv) {
  pdl_trigger();
  pdl_wait();
  __shared__ long long s_part[8];
  const int tid = threadIdx.x;
  long long c_sum = 0;
  for (int e = tid; e < E; e += 256) c_sum += counts[e];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c_sum += __shfl_xor_sync(0xffffffffu, c_sum, o);
  if ((tid & 31) == 0) s_part[tid >> 5] = c_sum;
  __syncthreads();
  long long total_i = 0;
#pragma unroll
  for (int w = 0; w < 8; ++w) total_i += s_part[w];
  // sum of counts in fp32 (exact below 2^24 pairs), clamped below at 1
  const float total = fmaxf(__ll2float_rn(total_i), 1.0f);
  for (int e = tid; e < E; e += 256) {
    const float p = __fdiv_rn(__int2float_rn(counts[e]), total);
    float err = __fsub_rn(target, p);
    if (p < thresh) err = __fadd_rn(err, starved_add);
    const float b = __fadd_rn(bias[e], __fmul_rn(err, rate));
    bias[e] = fminf(fmaxf(b, -clampv), clampv);
  }
}

// noaux_tc-style update (SpecForge PR #931, "What to watch": a fixed step
// per micro-batch): bias_e += rate * sign(mean(c) - c_e), fp32.
__global__ void __launch_bounds__(256)
bias_update_sign_kernel(const int32_t* __restrict__ counts, float* __restrict__ bias, int E,
                        float rate) {
  pdl_trigger();
  pdl_wait();
  __shared__ long long s_part[8];
  const int tid = threadIdx.x;
  long long c_sum = 0;
  for (int e = tid; e < E; e += 256) c_sum += counts[e];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c_sum += __shfl_xor_sync(0xffffffffu, c_sum, o);
  if ((tid & 31) == 0) s_part[tid >> 5] = c_sum;
  __syncthreads();
  long long total_i = 0;
#pragma unroll
  for (int w = 0; w < 8; ++w) total_i += s_part[w];
  const float mean = __fdiv_rn(__ll2float_rn(total_i), __int2float_rn(E));
  for (int e = tid; e < E; e += 256) {
    const float d = __fsub_rn(mean, __int2float_rn(counts[e]));
    const float step = d > 0.f ? rate : (d < 0.f ? -rate : 0.f);
    bias[e] = __fadd_rn(bias[e], step);
  }
}

}  // namespace

template <bool BF16>
cudaError_t launch_combine(dim3 grid, int threads, cudaStream_t stream, const uint4* y,
                           const int32_t* sp, const float* w, const uint4* ysh, uint4* out, int T,
                           int vecs, int k) {
  const dim3 block(threads);
  switch (k) {
    case 1:
      return launch_pdl(combine_kernel<BF16, 1>, grid, block, 0, stream, y, sp, w, ysh, out, T,
                        vecs, k);
    case 2:
      return launch_pdl(combine_kernel<BF16, 2>, grid, block, 0, stream, y, sp, w, ysh, out, T,
                        vecs, k);
    case 4:
      return launch_pdl(combine_kernel<BF16, 4>, grid, block, 0, stream, y, sp, w, ysh, out, T,
                        vecs, k);
    case 6:
      return launch_pdl(combine_kernel<BF16, 6>, grid, block, 0, stream, y, sp, w, ysh, out, T,
                        vecs, k);
    case 8:
      return launch_pdl(combine_kernel<BF16, 8>, grid, block, 0, stream, y, sp, w, ysh, out, T,
                        vecs, k);
    default:
      return launch_pdl(combine_kernel<BF16, 0>, grid, block, 0, stream, y, sp, w, ysh, out, T,
                        vecs, k);
  }
}

cudaError_t combine(bool bf16, const void* y_perm, const int32_t* slot_pos, const float* topk_w,
                    const void* y_shared, void* out, int T, int d, int k, cudaStream_t stream) {
  const int vecs = d * (bf16 ? 2 : 4) / 16;
  const int warps = 8;
  const dim3 grid((T + warps - 1) / warps);
  const uint4* y = static_cast<const uint4*>(y_perm);
  const uint4* ysh = static_cast<const uint4*>(y_shared);
  uint4* o = static_cast<uint4*>(out);
  if (bf16)
    return launch_combine<true>(grid, warps * 32, stream, y, slot_pos, topk_w, ysh, o, T, vecs, k);
  return launch_combine<false>(grid, warps * 32, stream, y, slot_pos, topk_w, ysh, o, T, vecs, k);
}

cudaError_t bias_update(const int32_t* counts, float* bias, int E, float target, float thresh,
                        float starved_add, float rate, float clamp, cudaStream_t stream) {
  return launch_pdl(bias_update_kernel, dim3(1), dim3(256), 0, stream, counts, bias, E, target,
                    thresh, starved_add, rate, clamp);
}

cudaError_t bias_update_sign(const int32_t* counts, float* bias, int E, float rate,
                             cudaStream_t stream) {
  return launch_pdl(bias_update_sign_kernel, dim3(1), dim3(256), 0, stream, counts, bias, E, rate);
}

}  // namespace moe
