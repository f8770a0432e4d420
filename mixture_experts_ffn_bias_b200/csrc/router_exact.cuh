// Exact re-decision of a router token whose fp32 selection keys hold a near
// tie (two of its top-(k+1) keys closer than the router's margin).
//
// The experts to decide over are the token's candidates (every expert whose
// fp32 key was within the margin of its (k+1)-th pick, which must contain the
// exact top-k) or all experts.  Their exact logits are fp64 sums of exact
// bf16 x bf16 products.  Selection uses the fp64 keys (ties to the lower
// expert id); the weights are formed in fp32 from the exact logits.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace moe {
namespace {

constexpr int kMaxPerLane = 8;   // E <= 256 = 8 x 32

// Decision on exact logits s_l[0..n) of experts s_e[0..n) (shared memory),
// written to idx_row / w_row.
__device__ void refine_select(const double* s_l, const int* s_e, int n, const float* bias,
                              int k, int gate, int renorm, bool all_experts, int space,
                              const float* noise_row, int32_t* idx_row, float* w_row) {
  const int lane = threadIdx.x & 31;
  double key[kMaxPerLane];
  float lf[kMaxPerLane];
  int ex[kMaxPerLane];
  bool taken[kMaxPerLane];
  float m = -INFINITY;
#pragma unroll
  for (int j = 0; j < kMaxPerLane; ++j) {
    const int c = lane + 32 * j;
    taken[j] = c >= n;
    ex[j] = c < n ? s_e[c] : 0x7fffffff;
    const double l = c < n ? s_l[c] : -INFINITY;
    lf[j] = static_cast<float>(l);
    key[j] = l;
    m = fmaxf(m, lf[j]);
  }
  if (space) {   // key base = the exact gate score (softmax: all experts are here)
    if (gate == 1) {
#pragma unroll
      for (int j = 0; j < kMaxPerLane; ++j) key[j] = 1.0 / (1.0 + exp(-key[j]));
    } else {
      double mm = -INFINITY, sum = 0.0;
#pragma unroll
      for (int j = 0; j < kMaxPerLane; ++j) mm = fmax(mm, key[j]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mm = fmax(mm, __shfl_xor_sync(0xffffffffu, mm, o));
#pragma unroll
      for (int j = 0; j < kMaxPerLane; ++j) {
        key[j] = exp(key[j] - mm);   // 0 past n
        sum += key[j];
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
#pragma unroll
      for (int j = 0; j < kMaxPerLane; ++j) key[j] = key[j] / sum;
    }
  }
#pragma unroll
  for (int j = 0; j < kMaxPerLane; ++j) {
    const int c = lane + 32 * j;
    key[j] = c < n ? key[j] + (bias ? static_cast<double>(bias[ex[j]]) : 0.0) +
                         (noise_row ? static_cast<double>(noise_row[ex[j]]) : 0.0)
                   : -INFINITY;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float S = 1.0f;
  if (gate == 0 && all_experts) {
    S = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxPerLane; ++j)
      if (lane + 32 * j < n) S += expf(lf[j] - m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) S += __shfl_xor_sync(0xffffffffu, S, o);
  }
  int my_idx = 0;
  float my_s = 0.f, ssum = 0.f;
  for (int j = 0; j < k; ++j) {
    double bk = -INFINITY;
    int be = 0x7fffffff, bslot = 0;
#pragma unroll
    for (int q = 0; q < kMaxPerLane; ++q) {
      if (!taken[q] && (key[q] > bk || (key[q] == bk && ex[q] < be))) {
        bk = key[q];
        be = ex[q];
        bslot = q;
      }
    }
    int owner = lane;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const double ok = __shfl_xor_sync(0xffffffffu, bk, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      const int ow = __shfl_xor_sync(0xffffffffu, owner, o);
      const int os = __shfl_xor_sync(0xffffffffu, bslot, o);
      if (ok > bk || (ok == bk && oe < be)) {
        bk = ok;
        be = oe;
        owner = ow;
        bslot = os;
      }
    }
    float l = 0.f;
#pragma unroll
    for (int q = 0; q < kMaxPerLane; ++q) {
      if (lane == owner && q == bslot) {
        taken[q] = true;
        l = lf[q];
      }
    }
    l = __shfl_sync(0xffffffffu, l, owner);
    const float sc = gate == 1 ? 1.0f / (1.0f + expf(-l)) : expf(l - m) / S;
    if (lane == j) {
      my_idx = be;
      my_s = sc;
    }
    ssum += sc;
  }
  if (lane < k) {
    idx_row[lane] = my_idx;
    w_row[lane] = renorm ? my_s / (ssum + 1e-9f) : my_s;
  }
}


}  // namespace
}  // namespace moe
