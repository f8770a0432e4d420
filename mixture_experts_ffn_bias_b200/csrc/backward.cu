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
//   sgemm_kernel        fp32 CUDA-core GEMM for the router gradients (the
//                       router runs in fp32: "moe-200m-qwen3-100b" README,
//                       "Per-layer numerics")
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
// A(m, k) = a[m * lda + k] (A_T: a[k * lda + m]), fp32; B(k, n) = b[k * ldb + n], bf16.
// 128 x 128 tile per block, K in steps of 8 through shared memory, 256
// threads with an 8 x 8 register tile each (rows ty + 16 i, columns
// 4 tx + 64 j + q, so the shared-memory reads are float4 and conflict free).
// N a multiple of 128, any M and K (rows past M and k past the slice read
// as zero); kslice a multiple of 8.
constexpr int SG_T = 128, SG_K = 8;

template <bool A_T>
__global__ void __launch_bounds__(256)
sgemm_kernel(const float* __restrict__ a, int lda, const __nv_bfloat16* __restrict__ b, int ldb,
             int M, int N, int K, int kslice, float* __restrict__ part) {
  pdl_trigger();
  pdl_wait();
  __shared__ __align__(16) float As[SG_K][SG_T];
  __shared__ __align__(16) float Bs[SG_K][SG_T];
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int m0 = blockIdx.y * SG_T, n0 = blockIdx.x * SG_T;
  const int kbeg = blockIdx.z * kslice, kend = min(K, kbeg + kslice);
  const bool vec = (lda & 3) == 0;   // 16-byte aligned rows of A
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  for (int k0 = kbeg; k0 < kend; k0 += SG_K) {
    // A tile: 8 x 128 floats = 256 float4
    if (A_T) {
      const int kk = tid >> 5, mm = (tid & 31) * 4;   // row kk, columns mm..mm+3
      const int k = k0 + kk, m = m0 + mm;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (k < kend) {
        const float* src = a + static_cast<size_t>(k) * lda + m;
        if (vec && m + 3 < M) {
          v = *reinterpret_cast<const float4*>(src);
        } else {
          v.x = m < M ? src[0] : 0.f;
          v.y = m + 1 < M ? src[1] : 0.f;
          v.z = m + 2 < M ? src[2] : 0.f;
          v.w = m + 3 < M ? src[3] : 0.f;
        }
      }
      *reinterpret_cast<float4*>(&As[kk][mm]) = v;
    } else {
      const int mm = tid >> 1, kk = (tid & 1) * 4;     // row mm, k columns kk..kk+3
      const int m = m0 + mm, k = k0 + kk;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (m < M) {
        const float* src = a + static_cast<size_t>(m) * lda + k;
        if (vec && k + 3 < kend) {
          v = *reinterpret_cast<const float4*>(src);
        } else {
          v.x = k < kend ? src[0] : 0.f;
          v.y = k + 1 < kend ? src[1] : 0.f;
          v.z = k + 2 < kend ? src[2] : 0.f;
          v.w = k + 3 < kend ? src[3] : 0.f;
        }
      }
      As[kk][mm] = v.x;
      As[kk + 1][mm] = v.y;
      As[kk + 2][mm] = v.z;
      As[kk + 3][mm] = v.w;
    }
    // B tile: 8 x 128 bf16 = 128 x 16 bytes
    if (tid < 128) {
      const int kk = tid >> 4, nn = (tid & 15) * 8;
      const int k = k0 + kk, n = n0 + nn;
      float f[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (k < kend && n + 7 < N) {
        const uint4 u = *reinterpret_cast<const uint4*>(b + static_cast<size_t>(k) * ldb + n);
        unpack8(u, f);
      }
      *reinterpret_cast<float4*>(&Bs[kk][nn]) = make_float4(f[0], f[1], f[2], f[3]);
      *reinterpret_cast<float4*>(&Bs[kk][nn + 4]) = make_float4(f[4], f[5], f[6], f[7]);
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < SG_K; ++kk) {
      float av[8], bv[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) av[i] = As[kk][ty + 16 * i];
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[kk][4 * tx]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[kk][4 * tx + 64]);
      bv[0] = b0.x; bv[1] = b0.y; bv[2] = b0.z; bv[3] = b0.w;
      bv[4] = b1.x; bv[5] = b1.y; bv[6] = b1.z; bv[7] = b1.w;
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
  float* out = part + static_cast<size_t>(blockIdx.z) * M * N;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int m = m0 + ty + 16 * i;
    if (m >= M) continue;
    float* row = out + static_cast<size_t>(m) * N + n0 + 4 * tx;
    *reinterpret_cast<float4*>(row) = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
    *reinterpret_cast<float4*>(row + 64) =
        make_float4(acc[i][4], acc[i][5], acc[i][6], acc[i][7]);
  }
}

// out[i] = sum_z part[z][i] (fixed order)
__global__ void __launch_bounds__(256)
sum_slices_kernel(const float* __restrict__ part, int slices, long long n,
                  float* __restrict__ out) {
  pdl_trigger();
  pdl_wait();
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    float s = 0.f;
    for (int z = 0; z < slices; ++z) s += part[z * n + i];
    out[i] = s;
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

int sgemm_slices(int K) {
  int s = (K + 1023) / 1024;
  return s < 1 ? 1 : (s > 16 ? 16 : s);
}

cudaError_t sgemm_f32(bool a_t, const float* a, int lda, const void* b, int ldb, int M, int N,
                      int K, float* part, float* out, cudaStream_t stream) {
  if (N % SG_T || ldb % 8) return cudaErrorInvalidValue;
  const int slices = sgemm_slices(K);
  const int kslice = ((K + slices - 1) / slices + SG_K - 1) / SG_K * SG_K;
  const dim3 grid(N / SG_T, (M + SG_T - 1) / SG_T, slices);
  if (slices == 1) part = out;   // one slice: the partial sum is the result
  cudaError_t e =
      a_t ? launch_pdl(sgemm_kernel<true>, grid, dim3(256), 0, stream, a, lda,
                       static_cast<const __nv_bfloat16*>(b), ldb, M, N, K, kslice, part)
          : launch_pdl(sgemm_kernel<false>, grid, dim3(256), 0, stream, a, lda,
                       static_cast<const __nv_bfloat16*>(b), ldb, M, N, K, kslice, part);
  if (e != cudaSuccess || slices == 1) return e;
  const long long n = static_cast<long long>(M) * N;
  return launch_pdl(sum_slices_kernel, dim3(grid_1d(n)), dim3(256), 0, stream, part, slices, n,
                    out);
}

}  // namespace moe
