// Backward pass of the MoE layer: the memory-bound steps and the fp32 router
// gradient.  The contractions of the experts run on the tensor cores (the
// grouped GEMM of grouped_gemm_sm100.cu for dH and dX and for the recomputed
// gate/up pass whose epilogue forms dG and dU, the K-grouped GEMM of
// grouped_gemm_wgrad_sm100.cu for the weight gradients); this file holds
// what feeds and finishes them:
//   bwd_dy_kernel       dw[t, j] = <dout[t], y_perm[slot]>, dY[slot] = w[t, j] dout[t]
//   dx_gather_kernel    dx[t] = sum_j dX[slot(t, j)] + dx_router[t] (+ dx_shared[t])
//   router_dlogits_kernel  dlogits from dw through the (renormalised) gate
//   router_grad_split_kernel  dlogits (fp32) as three bf16 terms, in the two
//                       layouts the router-gradient GEMMs read (the router
//                       runs in fp32: "moe-200m-qwen3-100b" README,
//                       "Per-layer numerics")
//   router_grad_reduce_kernel  dW_router = sum of the per-slice, per-term
//                       fp32 partial products, in a fixed order
// The chain rule is that of the layer in the "moe-200m-qwen3-100b" README
// ("Architecture diagram", SigmoidRouter forward): out = shared(x) +
// sum_j w_j expert_j(x), w = gate scores of the picked experts, renormalised.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.h"
#include "launch.cuh"

namespace moe {
namespace {

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
  const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&u);
#pragma unroll
  for (int i = 0; i < 8; ++i) f[i] = __bfloat162float(h[i]);
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  uint4 o;
  uint32_t* p = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 v = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    p[i] = *reinterpret_cast<uint32_t*>(&v);
  }
  return o;
}

// One warp per token.  oct = d / 8 (uint4 of 8 bf16 per lane step).  Lane j
// holds the slot and weight of the token's j-th pair; the dout row is read
// once, four 16-byte pieces per lane at a time, and each pair's y_perm
// pieces are all requested before they are used.
__global__ void __launch_bounds__(256)
bwd_dy_kernel(const uint4* __restrict__ dout, const uint4* __restrict__ y_perm,
              const int32_t* __restrict__ slot_pos, const float* __restrict__ topk_w,
              uint4* __restrict__ dy, float* __restrict__ dw, int T, int oct, int k) {
  pdl_trigger();
  pdl_wait();
  constexpr int U = 4;
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  int my_slot = -1;
  float my_w = 0.f;
  if (lane < k) {
    my_slot = slot_pos[static_cast<size_t>(t) * k + lane];
    my_w = topk_w[static_cast<size_t>(t) * k + lane];
  }
  const uint4* drow = dout + static_cast<size_t>(t) * oct;
  float my_dot = 0.f;   // lane j: <dout[t], y_perm[slot j]>
  for (int c0 = lane; c0 < oct; c0 += 32 * U) {
    float a[U][8];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = c0 + 32 * u;
      if (c < oct) unpack8(__ldg(drow + c), a[u]);
    }
    for (int j = 0; j < k; ++j) {
      const int r = __shfl_sync(0xffffffffu, my_slot, j);
      const float w = __shfl_sync(0xffffffffu, my_w, j);
      if (r < 0) continue;
      const uint4* yrow = y_perm + static_cast<size_t>(r) * oct;
      uint4* dyrow = dy + static_cast<size_t>(r) * oct;
      uint4 yv[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c = c0 + 32 * u;
        yv[u] = c < oct ? __ldcs(yrow + c) : make_uint4(0u, 0u, 0u, 0u);
      }
      float dot = 0.f;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c = c0 + 32 * u;
        if (c >= oct) continue;
        float b[8], o[8];
        unpack8(yv[u], b);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          dot = fmaf(a[u][i], b[i], dot);
          o[i] = w * a[u][i];
        }
        dyrow[c] = pack8(o);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      if (lane == j) my_dot += dot;
    }
  }
  if (lane < k) dw[static_cast<size_t>(t) * k + lane] = my_slot < 0 ? 0.f : my_dot;
}

// One warp per token: dx = sum_j dX[slot] + dxr (fp32) + dxs (bf16, may be
// null).  Lane j holds the slot of the token's j-th pair; for each 16-byte
// piece of the row all k rows are requested before they are added (pairs in
// j order, k <= 32).
__global__ void __launch_bounds__(256)
dx_gather_kernel(const uint4* __restrict__ dxp, const int32_t* __restrict__ slot_pos,
                 const float4* __restrict__ dxr, const uint4* __restrict__ dxs,
                 uint4* __restrict__ dx, int T, int oct, int k) {
  pdl_trigger();
  pdl_wait();
  constexpr int KB = 8;   // rows requested together
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  const int my_slot = lane < k ? slot_pos[static_cast<size_t>(t) * k + lane] : -1;
  for (int c = lane; c < oct; c += 32) {
    float acc[8];
    const float4 a = dxr[(static_cast<size_t>(t) * oct + c) * 2];
    const float4 b = dxr[(static_cast<size_t>(t) * oct + c) * 2 + 1];
    acc[0] = a.x; acc[1] = a.y; acc[2] = a.z; acc[3] = a.w;
    acc[4] = b.x; acc[5] = b.y; acc[6] = b.z; acc[7] = b.w;
    if (dxs) {
      float s[8];
      unpack8(dxs[static_cast<size_t>(t) * oct + c], s);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += s[i];
    }
    for (int j0 = 0; j0 < k; j0 += KB) {
      uint4 v[KB];
#pragma unroll
      for (int q = 0; q < KB; ++q) {
        const int r = __shfl_sync(0xffffffffu, my_slot, (j0 + q) & 31);
        v[q] = (j0 + q < k && r >= 0) ? __ldcs(dxp + static_cast<size_t>(r) * oct + c)
                                      : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int q = 0; q < KB; ++q) {
        float f[8];
        unpack8(v[q], f);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] += f[i];
      }
    }
    dx[static_cast<size_t>(t) * oct + c] = pack8(acc);
  }
}

constexpr int kMaxLane = 8;   // E <= 256

// One warp per token.  logits [T, E] fp32 (no offset), offset [E] or null.
__global__ void __launch_bounds__(256)
router_dlogits_kernel(const float* __restrict__ logits, const float* __restrict__ offset,
                      const int32_t* __restrict__ topk_idx, const float* __restrict__ topk_w,
                      const float* __restrict__ dw, int T, int E, int k, int gate, int renorm,
                      float* __restrict__ dlogits) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  float s[kMaxLane], ds[kMaxLane];
  float lmax = -INFINITY;
#pragma unroll
  for (int i = 0; i < kMaxLane; ++i) {
    const int e = lane + 32 * i;
    s[i] = e < E ? logits[static_cast<size_t>(t) * E + e] + (offset ? offset[e] : 0.f)
                 : -INFINITY;
    lmax = fmaxf(lmax, s[i]);
    ds[i] = 0.f;
  }
  if (gate == 1) {
#pragma unroll
    for (int i = 0; i < kMaxLane; ++i) s[i] = 1.0f / (1.0f + expf(-s[i]));   // 0 past E
  } else {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lmax = fmaxf(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < kMaxLane; ++i) {
      s[i] = expf(s[i] - lmax);
      sum += s[i];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
#pragma unroll
    for (int i = 0; i < kMaxLane; ++i) s[i] /= sum;
  }
  // the picked experts' scores, their sum and sum_j dw_j w_j
  float ssel = 0.f, dsum = 0.f;
  for (int j = 0; j < k; ++j) {
    const size_t p = static_cast<size_t>(t) * k + j;
    const int e = topk_idx[p];
    float se = 0.f;
#pragma unroll
    for (int i = 0; i < kMaxLane; ++i)
      if (lane + 32 * i == e) se = s[i];
    se = __shfl_sync(0xffffffffu, se, e & 31);
    ssel += se;
    dsum += dw[p] * topk_w[p];
  }
  for (int j = 0; j < k; ++j) {
    const size_t p = static_cast<size_t>(t) * k + j;
    const int e = topk_idx[p];
    const float g = renorm ? (dw[p] - dsum) / (ssel + 1e-9f) : dw[p];
#pragma unroll
    for (int i = 0; i < kMaxLane; ++i)
      if (lane + 32 * i == e) ds[i] += g;
  }
  float dot = 0.f;
  if (gate == 0) {
#pragma unroll
    for (int i = 0; i < kMaxLane; ++i) dot += ds[i] * s[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
  }
#pragma unroll
  for (int i = 0; i < kMaxLane; ++i) {
    const int e = lane + 32 * i;
    if (e < E)
      dlogits[static_cast<size_t>(t) * E + e] =
          gate == 1 ? ds[i] * s[i] * (1.0f - s[i]) : s[i] * (ds[i] - dot);
  }
}

// fp32 CUDA-core GEMM, split over K: part[z][m][n] = sum_{k in slice z} A(m, k) B(k, n).
// x's rows in expert order, for a forward that gathered them instead of
// writing x_perm (flag set): x_perm[r] = x[perm_src[r]], one warp per row
// (grid-stride); a row whose source is out of range (a skipped pair) is
// zeroed.  With the flag clear the forward's x_perm is already there and
// nothing is done.
__global__ void __launch_bounds__(256)
fill_xperm_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ perm_src,
                  const uint32_t* __restrict__ flag, uint4* __restrict__ x_perm, long long R,
                  int T, int vecs) {
  pdl_trigger();
  pdl_wait();
  if (*flag == 0u) return;
  const int lane = threadIdx.x & 31;
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  for (long long r = blockIdx.x * static_cast<long long>(blockDim.x >> 5) + (threadIdx.x >> 5);
       r < R; r += warps) {
    const int t = perm_src[r];
    const bool ok = t >= 0 && t < T;
    uint4* dst = x_perm + r * vecs;
    const uint4* src = x + static_cast<long long>(ok ? t : 0) * vecs;
    for (int c = lane; c < vecs; c += 32)
      dst[c] = ok ? __ldg(src + c) : make_uint4(0u, 0u, 0u, 0u);
  }
}

// The router gradients dW_router = dlogits^T x and dx_router = dlogits Wr
// run on the tensor cores.  x and Wr are bf16; dlogits (fp32) is written as
// h1 + h2 + h3 with h1 = bf16(v), h2 = bf16(v - h1), h3 = bf16(v - h1 - h2)
// (each difference exact in fp32), which represents v to within fp32
// rounding (2^-24 relative); every product with a bf16 value is exact in
// fp32, so the tensor cores' fp32 sums are the rounding, as in an fp32 GEMM.  Term j of expert e sits at index
// j * Ep + e (Ep = E rounded up to 64, zeros past E):
//   adx [T, 3 Ep]            row t: the terms of dlogits[t, :]   (dx GEMM, K = 3 Ep)
//   adw [G, 3 Ep, Ks]        slice g of the tokens, transposed:  (dW GEMM, K = Ks
//                            per slice, zeros past T)
// goff[g] = g * 3 Ep are the row groups of adw (one GEMM group per slice).
// Block b takes tokens [32 b, 32 b + 32), which lie in one slice.
__global__ void __launch_bounds__(256)
router_grad_split_kernel(const float* __restrict__ dlogits, int T, int E, int Ep, int Ks, int G,
                         __nv_bfloat16* __restrict__ adx, __nv_bfloat16* __restrict__ adw,
                         int32_t* __restrict__ goff) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ float s_v[];            // [32][E + 1]
  const int ld = E + 1;
  const int t0 = blockIdx.x * 32;
  if (blockIdx.x == 0)
    for (int g = threadIdx.x; g <= G; g += blockDim.x) goff[g] = g * 3 * Ep;
  for (int i = threadIdx.x; i < 32 * E; i += blockDim.x) {
    const int r = i / E, e = i - r * E;
    s_v[r * ld + e] = t0 + r < T ? dlogits[static_cast<size_t>(t0 + r) * E + e] : 0.f;
  }
  __syncthreads();
  const int C3 = 3 * Ep;
  auto term = [](float v, int j) {
    const __nv_bfloat16 h1 = __float2bfloat16_rn(v);
    const float r1 = v - __bfloat162float(h1);
    if (j == 0) return h1;
    const __nv_bfloat16 h2 = __float2bfloat16_rn(r1);
    if (j == 1) return h2;
    return __float2bfloat16_rn(r1 - __bfloat162float(h2));
  };
  // 16-byte stores of eight terms: eight experts of one token (adx; Ep is a
  // multiple of 64, so the eight share the term j), eight tokens of one
  // expert (adw)
  const int c8n = C3 / 8;
  for (int i = threadIdx.x; i < 32 * c8n; i += blockDim.x) {
    const int r = i / c8n, c = (i - r * c8n) * 8;
    if (t0 + r >= T) continue;
    const int j = c / Ep, e0 = c - j * Ep;
    __align__(16) __nv_bfloat16 h[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) h[q] = term(e0 + q < E ? s_v[r * ld + e0 + q] : 0.f, j);
    *reinterpret_cast<uint4*>(adx + static_cast<size_t>(t0 + r) * C3 + c) =
        *reinterpret_cast<const uint4*>(h);
  }
  const int g = t0 / Ks, k0 = t0 - g * Ks;
  for (int i = threadIdx.x; i < C3 * 4; i += blockDim.x) {
    const int row = i >> 2, r0 = (i & 3) * 8;
    const int j = row / Ep, e = row - j * Ep;
    __align__(16) __nv_bfloat16 h[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) h[q] = term(e < E ? s_v[(r0 + q) * ld + e] : 0.f, j);
    *reinterpret_cast<uint4*>(adw + (static_cast<size_t>(g) * C3 + row) * Ks + k0 + r0) =
        *reinterpret_cast<const uint4*>(h);
  }
}

// out[e, n] = sum_g sum_j part[g * 3 Ep + j * Ep + e, n]  (g, then j: a fixed
// order)
__global__ void __launch_bounds__(256)
router_grad_reduce_kernel(const float* __restrict__ part, int G, int E, int Ep, int d,
                          float* __restrict__ out) {
  pdl_trigger();
  pdl_wait();
  const long long n = static_cast<long long>(E) * d;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long e = i / d, c = i - e * d;
    float acc = 0.f;
    for (int g = 0; g < G; ++g)
      for (int j = 0; j < 3; ++j)
        acc += part[(static_cast<long long>(g) * 3 * Ep + j * Ep + e) * d + c];
    out[i] = acc;
  }
}

int grid_1d(long long n) {
  const long long b = (n + 255) / 256;
  return static_cast<int>(b < 4096 ? (b > 0 ? b : 1) : 4096);
}

}  // namespace

cudaError_t bwd_dy(const void* dout, const void* y_perm, const int32_t* slot_pos,
                   const float* topk_w, void* dy, float* dw, int T, int d, int k,
                   cudaStream_t stream) {
  const int warps = 8;
  return launch_pdl(bwd_dy_kernel, dim3((T + warps - 1) / warps), dim3(warps * 32), 0, stream,
                    static_cast<const uint4*>(dout), static_cast<const uint4*>(y_perm), slot_pos,
                    topk_w, static_cast<uint4*>(dy), dw, T, d / 8, k);
}

cudaError_t dx_gather(const void* dxp, const int32_t* slot_pos, const float* dxr, const void* dxs,
                      void* dx, int T, int d, int k, cudaStream_t stream) {
  const int warps = 8;
  return launch_pdl(dx_gather_kernel, dim3((T + warps - 1) / warps), dim3(warps * 32), 0, stream,
                    static_cast<const uint4*>(dxp), slot_pos, reinterpret_cast<const float4*>(dxr),
                    static_cast<const uint4*>(dxs), static_cast<uint4*>(dx), T, d / 8, k);
}

cudaError_t router_dlogits(const float* logits, const float* offset, const int32_t* topk_idx,
                           const float* topk_w, const float* dw, int T, int E, int k, int gate,
                           int renorm, float* dlogits, cudaStream_t stream) {
  const int warps = 8;
  return launch_pdl(router_dlogits_kernel, dim3((T + warps - 1) / warps), dim3(warps * 32), 0,
                    stream, logits, offset, topk_idx, topk_w, dw, T, E, k, gate, renorm,
                    dlogits);
}

cudaError_t fill_xperm(const void* x, const int32_t* perm_src, const uint32_t* flag,
                       void* x_perm, long long R, int T, int d, cudaStream_t stream) {
  const int warps = 8;
  long long blocks = (R + warps - 1) / warps;
  if (blocks > 1184) blocks = 1184;   // 8 per SM; rows are taken grid-stride
  if (blocks < 1) blocks = 1;
  return launch_pdl(fill_xperm_kernel, dim3(static_cast<unsigned>(blocks)), dim3(warps * 32), 0,
                    stream, static_cast<const uint4*>(x), perm_src, flag,
                    static_cast<uint4*>(x_perm), R, T, d / 8);
}

RouterGradShape router_grad_shape(int T, int E) {
  RouterGradShape r;
  r.Ep = (E + 63) / 64 * 64;
  // token slices of the dW GEMM: about 16, each a multiple of 64 tokens
  r.Ks = ((T + 15) / 16 + 63) / 64 * 64;
  if (r.Ks < 64) r.Ks = 64;
  r.G = (T + r.Ks - 1) / r.Ks;
  return r;
}

cudaError_t router_grad_split(const float* dlogits, int T, int E, const RouterGradShape& r,
                              void* adx, void* adw, int32_t* goff, cudaStream_t stream) {
  const size_t smem = static_cast<size_t>(32) * (E + 1) * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(router_grad_split_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  // every column of every slice is written, zeros past T
  const int blocks = r.G * r.Ks / 32;
  return launch_pdl(router_grad_split_kernel, dim3(blocks), dim3(256), smem, stream, dlogits, T,
                    E, r.Ep, r.Ks, r.G, static_cast<__nv_bfloat16*>(adx),
                    static_cast<__nv_bfloat16*>(adw), goff);
}

cudaError_t router_grad_reduce(const float* part, const RouterGradShape& r, int E, int d,
                               float* out, cudaStream_t stream) {
  const long long n = static_cast<long long>(E) * d;
  return launch_pdl(router_grad_reduce_kernel, dim3(grid_1d(n)), dim3(256), 0, stream, part,
                    r.G, E, r.Ep, d, out);
}

}  // namespace moe
