// Backward pass of the MoE layer: the memory-bound steps and the fp32 router
// gradient.  The contractions of the experts run on the tensor cores (the
// plain grouped GEMM of grouped_gemm_sm100.cu for dH and dX, the K-grouped
// GEMM of grouped_gemm_wgrad_sm100.cu for the weight gradients); this file
// holds what feeds and finishes them:
//   bwd_dy_kernel       dw[t, j] = <dout[t], y_perm[slot]>, dY[slot] = w[t, j] dout[t]
//   gtranspose_kernel   rows of each group -> padded columns (the K-grouped
//                       operands), zeros in the padding
//   pad_offsets_kernel  padded column offsets of the groups
//   swiglu_bwd_kernel   dG = dH * U * silu'(G), dU = dH * silu(G)
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

// One warp per token.  oct = d / 8 (uint4 of 8 bf16 per lane step).
__global__ void __launch_bounds__(256)
bwd_dy_kernel(const uint4* __restrict__ dout, const uint4* __restrict__ y_perm,
              const int32_t* __restrict__ slot_pos, const float* __restrict__ topk_w,
              uint4* __restrict__ dy, float* __restrict__ dw, int T, int oct, int k) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  const uint4* drow = dout + static_cast<size_t>(t) * oct;
  for (int j = 0; j < k; ++j) {
    const size_t p = static_cast<size_t>(t) * k + j;
    const int r = slot_pos[p];
    if (r < 0) {
      if (lane == 0) dw[p] = 0.f;
      continue;
    }
    const float w = topk_w[p];
    const uint4* yrow = y_perm + static_cast<size_t>(r) * oct;
    uint4* dyrow = dy + static_cast<size_t>(r) * oct;
    float dot = 0.f;
    for (int c = lane; c < oct; c += 32) {
      float a[8], b[8], o[8];
      unpack8(drow[c], a);
      unpack8(__ldcs(yrow + c), b);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        dot = fmaf(a[i], b[i], dot);
        o[i] = w * a[i];
      }
      dyrow[c] = pack8(o);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    if (lane == 0) dw[p] = dot;
  }
}

// Transposes move 64 x 64 bf16 tiles through shared memory: 16-byte global
// loads of the source rows (a warp reads four full 128-byte rows), and
// 128-byte output rows written as bf16 pairs by a warp.  The tile's rows are
// 66 elements apart (33 words), so the column reads hit at most two lanes
// per bank.  All dimensions here are multiples of 64 (bf16 layers have d, F
// multiples of 128; padded column counts are multiples of 64).
constexpr int TT = 64;
constexpr int TROW = TT + 2;

// Loads source rows src_row(i), i < 64 (negative: zeros), columns [c0, c0+64).
__device__ __forceinline__ void load_tile(uint16_t (*tile)[TROW], const __nv_bfloat16* in,
                                          int cols, int c0, const int* src_row) {
  for (int idx = threadIdx.x; idx < TT * 8; idx += blockDim.x) {
    const int i = idx >> 3, v = idx & 7;
    const int src = src_row[i];
    uint4 u = make_uint4(0u, 0u, 0u, 0u);
    if (src >= 0)
      u = *reinterpret_cast<const uint4*>(in + static_cast<size_t>(src) * cols + c0 + v * 8);
    uint32_t* t = reinterpret_cast<uint32_t*>(&tile[i][v * 8]);
    t[0] = u.x; t[1] = u.y; t[2] = u.z; t[3] = u.w;
  }
}

// Writes out[(c0 + c) * ldo + base + i] = tile[i][c] for c, i < 64.
__device__ __forceinline__ void store_tile_t(const uint16_t (*tile)[TROW], __nv_bfloat16* out,
                                             long long ldo, long long base, int c0) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int c = warp; c < TT; c += nw) {
    const uint32_t lo = tile[2 * lane][c], hi = tile[2 * lane + 1][c];
    reinterpret_cast<uint32_t*>(out + (c0 + c) * ldo + base)[lane] = lo | (hi << 16);
  }
}

// out[b][c][col_off + r] = in[b][r][c] for r < rows, c < cols.
// Padded column offsets: poff[g + 1] = poff[g] + roundup(rows_g, 64).
// offsets null: one group of rows_single rows.
__global__ void pad_offsets_kernel(const int32_t* __restrict__ offsets, int G, int rows_single,
                                   int32_t* __restrict__ poff) {
  pdl_trigger();
  pdl_wait();
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  int run = 0;
  poff[0] = 0;
  for (int g = 0; g < G; ++g) {
    const int rows = offsets ? offsets[g + 1] - offsets[g] : rows_single;
    run += (rows + 63) / 64 * 64;
    poff[g + 1] = run;
  }
}

// out [cols, kp]: column p of out is row src(p) of in [rows, cols], where
// p = poff[g] + i < poff[g] + rows_g maps to row offsets[g] + i (gathered
// through `gather` when not null), and every other p is zero.  The grid
// covers kp x cols in 64 x 64 tiles; the group offsets are staged in shared
// memory for the per-position search.
__global__ void __launch_bounds__(256)
gtranspose_kernel(const __nv_bfloat16* __restrict__ in, int cols,
                  const int32_t* __restrict__ offsets, int G, int rows_single,
                  const int32_t* __restrict__ poff, const int32_t* __restrict__ gather,
                  __nv_bfloat16* __restrict__ out, int kp) {
  pdl_trigger();
  pdl_wait();
  __shared__ __align__(16) uint16_t tile[TT][TROW];
  __shared__ int s_poff[258];
  __shared__ int s_off[258];
  __shared__ int s_src[TT];
  const int p0 = blockIdx.x * TT, c0 = blockIdx.y * TT;
  for (int g = threadIdx.x; g <= G; g += blockDim.x) {
    s_poff[g] = poff[g];
    s_off[g] = offsets ? offsets[g] : (g == 0 ? 0 : rows_single);
  }
  __syncthreads();
  if (threadIdx.x < TT) {
    const int p = p0 + static_cast<int>(threadIdx.x);
    int src = -1;
    if (p < s_poff[G]) {
      int lo = 0, hi = G - 1;   // last g with poff[g] <= p
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_poff[mid] <= p) lo = mid; else hi = mid - 1;
      }
      const int i = p - s_poff[lo];
      if (i < s_off[lo + 1] - s_off[lo]) src = gather ? gather[s_off[lo] + i] : s_off[lo] + i;
    }
    s_src[threadIdx.x] = src;
  }
  __syncthreads();
  load_tile(tile, in, cols, c0, s_src);
  __syncthreads();
  store_tile_t(tile, out, kp, p0, c0);
}

// dGU [n, 2F]: columns [0, F) = dG, [F, 2F) = dU; G, U, dH [n, F].  fq = F / 8.
__global__ void __launch_bounds__(256)
swiglu_bwd_kernel(const uint4* __restrict__ G, const uint4* __restrict__ U,
                  const uint4* __restrict__ dH, uint4* __restrict__ dGU, long long n8, int fq) {
  pdl_trigger();
  pdl_wait();
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long r = i / fq;
    const int c = static_cast<int>(i - r * fq);
    float g[8], u[8], dh[8], dg[8], du[8];
    unpack8(G[i], g);
    unpack8(U[i], u);
    unpack8(dH[i], dh);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float s = 1.0f / (1.0f + expf(-g[q]));
      du[q] = dh[q] * g[q] * s;
      dg[q] = dh[q] * u[q] * (s * (1.0f + g[q] * (1.0f - s)));
    }
    dGU[r * 2 * fq + c] = pack8(dg);
    dGU[r * 2 * fq + fq + c] = pack8(du);
  }
}

// One warp per token: dx = sum_j dX[slot] + dxr (fp32) + dxs (bf16, may be null).
__global__ void __launch_bounds__(256)
dx_gather_kernel(const uint4* __restrict__ dxp, const int32_t* __restrict__ slot_pos,
                 const float4* __restrict__ dxr, const uint4* __restrict__ dxs,
                 uint4* __restrict__ dx, int T, int oct, int k) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
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
    for (int j = 0; j < k; ++j) {
      const int r = slot_pos[static_cast<size_t>(t) * k + j];
      if (r < 0) continue;
      float v[8];
      unpack8(dxp[static_cast<size_t>(r) * oct + c], v);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += v[i];
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
  for (int i = threadIdx.x; i < 32 * C3; i += blockDim.x) {
    const int r = i / C3, c = i - r * C3;
    if (t0 + r >= T) continue;
    const int j = c / Ep, e = c - j * Ep;
    adx[static_cast<size_t>(t0 + r) * C3 + c] = term(e < E ? s_v[r * ld + e] : 0.f, j);
  }
  const int g = t0 / Ks, k0 = t0 - g * Ks;
  for (int i = threadIdx.x; i < C3 * 32; i += blockDim.x) {
    const int row = i >> 5, r = i & 31;
    const int j = row / Ep, e = row - j * Ep;
    adw[(static_cast<size_t>(g) * C3 + row) * Ks + k0 + r] =
        term(e < E ? s_v[r * ld + e] : 0.f, j);
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

cudaError_t pad_offsets(const int32_t* offsets, int G, int rows_single, int32_t* poff,
                        cudaStream_t stream) {
  return launch_pdl(pad_offsets_kernel, dim3(1), dim3(32), 0, stream, offsets, G, rows_single,
                    poff);
}

cudaError_t gtranspose_bf16(const void* in, int cols, const int32_t* offsets, int G,
                            int rows_single, const int32_t* poff, const int32_t* gather,
                            void* out, int kp, cudaStream_t stream) {
  if (kp % TT || cols % TT || G > 257) return cudaErrorInvalidValue;
  const dim3 grid(kp / TT, cols / TT);
  return launch_pdl(gtranspose_kernel, grid, dim3(256), 0, stream,
                    static_cast<const __nv_bfloat16*>(in), cols, offsets, G, rows_single, poff,
                    gather, static_cast<__nv_bfloat16*>(out), kp);
}

cudaError_t swiglu_bwd(const void* G, const void* U, const void* dH, void* dGU, long long n,
                       int F, cudaStream_t stream) {
  const long long n8 = n * (F / 8);
  return launch_pdl(swiglu_bwd_kernel, dim3(grid_1d(n8)), dim3(256), 0, stream,
                    static_cast<const uint4*>(G), static_cast<const uint4*>(U),
                    static_cast<const uint4*>(dH), static_cast<uint4*>(dGU), n8, F / 8);
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
