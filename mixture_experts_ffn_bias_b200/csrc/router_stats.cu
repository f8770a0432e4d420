// Router losses and health metrics from the logits of a batch and its
// routing: the aux dict of SigmoidRouter.forward in the "moe-200m-qwen3-100b"
// README (z-loss, DeepSeek aux loss, per-expert counts, load CV, entropy of
// the mean scores in bits) and the load metrics of SpecForge PR #931 ("What
// to watch": moe/load_max_ratio, experts without tokens).
//
// Two deterministic passes: blocks of 64 tokens (one warp per token, a
// warp's lanes own distinct experts) write per-block partial sums in fp64;
// one block adds the partials in a fixed order and forms the scalars.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.h"
#include "launch.cuh"

namespace moe {
namespace {

constexpr int kStatTok = 64;     // tokens per partial block
constexpr int kMaxE = 256;

template <typename L>
__global__ void __launch_bounds__(256)
stats_partial_kernel(const L* __restrict__ logits, int T, int E, int gate,
                     const int32_t* __restrict__ topk_idx, int k,
                     double* __restrict__ partials) {
  pdl_trigger();
  pdl_wait();
  __shared__ float s_sc[8][kMaxE];
  __shared__ int s_cnt[kMaxE];
  __shared__ double s_z[8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int e = threadIdx.x; e < kMaxE; e += 256) s_cnt[e] = 0;
  for (int e = lane; e < kMaxE; e += 32) s_sc[warp][e] = 0.f;
  double z = 0.0;
  __syncthreads();
  for (int i = 0; i < kStatTok / 8; ++i) {
    const int t = blockIdx.x * kStatTok + warp * (kStatTok / 8) + i;
    if (t >= T) break;
    float l[8];
    float m = -INFINITY;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane + 32 * j;
      l[j] = e < E ? static_cast<float>(logits[static_cast<size_t>(t) * E + e]) : -INFINITY;
      m = fmaxf(m, l[j]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float S = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (lane + 32 * j < E) S += expf(l[j] - m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) S += __shfl_xor_sync(0xffffffffu, S, o);
    const double lse = static_cast<double>(m) + log(static_cast<double>(S));
    z += lse * lse;   // identical in every lane; lane 0's copy is kept
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane + 32 * j;
      if (e < E)
        s_sc[warp][e] += gate == 1 ? 1.0f / (1.0f + expf(-l[j])) : expf(l[j] - m) / S;
    }
    if (lane < k) {
      const int e = topk_idx[static_cast<size_t>(t) * k + lane];
      if (e >= 0 && e < E) atomicAdd(&s_cnt[e], 1);
    }
  }
  if (lane == 0) s_z[warp] = z;
  __syncthreads();
  double* out = partials + static_cast<size_t>(blockIdx.x) * (2 * E + 1);
  for (int e = threadIdx.x; e < E; e += 256) {
    double acc = 0.0;
#pragma unroll
    for (int w = 0; w < 8; ++w) acc += static_cast<double>(s_sc[w][e]);
    out[e] = acc;
    out[E + e] = static_cast<double>(s_cnt[e]);
  }
  if (threadIdx.x == 0) {
    double zz = 0.0;
    for (int w = 0; w < 8; ++w) zz += s_z[w];
    out[2 * E] = zz;
  }
}

// Fixed-order tree sum over 256 slots of shared memory (all threads call).
__device__ double block_sum(double* s, double v) {
  const int tid = threadIdx.x;
  s[tid] = v;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (tid < o) s[tid] += s[tid + o];
    __syncthreads();
  }
  const double r = s[0];
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(256)
stats_final_kernel(const double* __restrict__ partials, int nb, int T, int E,
                   float* __restrict__ out) {
  pdl_trigger();
  pdl_wait();
  __shared__ double s[256];
  const int e = threadIdx.x;
  double sc = 0.0, cnt = 0.0;
  if (e < E) {
    for (int b = 0; b < nb; ++b) {
      sc += partials[static_cast<size_t>(b) * (2 * E + 1) + e];
      cnt += partials[static_cast<size_t>(b) * (2 * E + 1) + E + e];
    }
  }
  double zsum = 0.0;
  if (e == 0)
    for (int b = 0; b < nb; ++b) zsum += partials[static_cast<size_t>(b) * (2 * E + 1) + 2 * E];
  const double Td = static_cast<double>(T);
  const double p = sc / Td;                       // mean score of expert e
  const double frac = cnt / Td;                   // one_hot mean over tokens
  const double aux = static_cast<double>(E) * block_sum(s, e < E ? frac * p : 0.0);
  const double csum = block_sum(s, e < E ? cnt : 0.0);
  const double mean_c = csum / E;
  const double var = block_sum(s, e < E ? (cnt - mean_c) * (cnt - mean_c) : 0.0) / (E - 1);
  const double pa = e < E ? fmax(p, 1e-9) : 0.0;
  const double pa_sum = block_sum(s, pa);
  const double q = pa / pa_sum;
  const double ent = -block_sum(s, e < E ? q * log(q) : 0.0) / log(2.0);
  // max count and number of unused experts
  s[e] = e < E ? cnt : -1.0;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (e < o) s[e] = fmax(s[e], s[e + o]);
    __syncthreads();
  }
  const double cmax = s[0];
  __syncthreads();
  const double unused = block_sum(s, (e < E && cnt == 0.0) ? 1.0 : 0.0);
  if (e == 0) {
    out[0] = static_cast<float>(zsum / Td);
    out[1] = static_cast<float>(aux);
    out[2] = static_cast<float>(E > 1 ? sqrt(var) / fmax(mean_c, 1.0) : __longlong_as_double(0x7ff8000000000000ll));
    out[3] = static_cast<float>(ent);
    out[4] = static_cast<float>(mean_c > 0.0 ? cmax / mean_c : 0.0);
    out[5] = static_cast<float>(unused / E);
    out[6] = 0.f;
    out[7] = 0.f;
  }
}

}  // namespace

int stats_blocks(int T) { return (T + kStatTok - 1) / kStatTok; }

cudaError_t router_stats(bool fp64_logits, const void* logits, int T, int E, int gate,
                         const int32_t* topk_idx, int k, double* partials, float* out,
                         cudaStream_t stream) {
  const int nb = stats_blocks(T);
  cudaError_t e =
      fp64_logits
          ? launch_pdl(stats_partial_kernel<double>, dim3(nb), dim3(256), 0, stream,
                       static_cast<const double*>(logits), T, E, gate, topk_idx, k, partials)
          : launch_pdl(stats_partial_kernel<float>, dim3(nb), dim3(256), 0, stream,
                       static_cast<const float*>(logits), T, E, gate, topk_idx, k, partials);
  if (e != cudaSuccess) return e;
  return launch_pdl(stats_final_kernel, dim3(1), dim3(256), 0, stream, partials, nb, T, E, out);
}

}  // namespace moe
