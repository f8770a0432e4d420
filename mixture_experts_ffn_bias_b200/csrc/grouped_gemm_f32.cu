// fp32 grouped SwiGLU experts on CUDA cores (the fp32 layer has no bf16
// operands for the tensor cores; it is the small correctness-scale layer).
//
// Same contract as the bf16 tensor-core path: for each group g with rows
// [off[g], off[g+1]) of A,
//   gate/up pass:  H[r, n] = silu(A[r] . W1[g][n]) * (A[r] . W3[g][n])
//   down pass:     Y[r, n] = A[r] . W2[g][n]
// with fp32 accumulation.  32 x 32 output tiles, 256 threads, 4 outputs each.
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.h"
#include "launch.cuh"

namespace moe {
namespace {

constexpr int TM = 32, TN = 32, TK = 32, MAXG = 257;

template <bool SWIGLU>
__global__ void __launch_bounds__(256)
grouped_gemm_f32_kernel(const float* __restrict__ A, const int32_t* __restrict__ offsets, int G,
                        int rows_single, const float* __restrict__ B0,
                        const float* __restrict__ B1, int N, int K, float* __restrict__ C) {
  pdl_trigger();
  pdl_wait();
  __shared__ int s_off[MAXG + 1];
  __shared__ int s_pref[MAXG + 1];
  __shared__ float As[TK][TM + 1];
  __shared__ float Bs0[TK][TN + 1];
  __shared__ float Bs1[TK][TN + 1];
  const int tid = threadIdx.x;
  if (offsets == nullptr) G = 1;
  if (tid == 0) {
    int run = 0;
    for (int g = 0; g <= G; ++g) {
      s_off[g] = offsets ? offsets[g] : (g == 0 ? 0 : rows_single);
      s_pref[g] = run;
      if (g < G) {
        const int rows = (offsets ? offsets[g + 1] - offsets[g] : rows_single);
        run += (rows > 0 ? rows + TM - 1 : 0) / TM;
      }
    }
  }
  __syncthreads();
  const int mt = blockIdx.x;
  if (mt >= s_pref[G]) return;
  int g = 0;
  while (g + 1 < G && s_pref[g + 1] <= mt) ++g;
  const int m0 = (mt - s_pref[g]) * TM;
  const int rows_g = s_off[g + 1] - s_off[g];
  const int n0 = blockIdx.y * TN;
  const int tr = tid >> 3;        // output row in tile
  const int tc = (tid & 7) * 4;   // first of 4 output columns
  float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
  const float* Ag = A + static_cast<size_t>(s_off[g]) * K;
  const float* B0g = B0 + static_cast<size_t>(g) * N * K;
  const float* B1g = SWIGLU ? B1 + static_cast<size_t>(g) * N * K : nullptr;
  for (int k0 = 0; k0 < K; k0 += TK) {
    for (int i = tid; i < TM * TK; i += 256) {
      const int r = i / TK, kk = i % TK;
      const int row = m0 + r, col = k0 + kk;
      As[kk][r] = (row < rows_g && col < K) ? Ag[static_cast<size_t>(row) * K + col] : 0.f;
      const int n = n0 + r;
      Bs0[kk][r] = (n < N && col < K) ? B0g[static_cast<size_t>(n) * K + col] : 0.f;
      if (SWIGLU) Bs1[kk][r] = (n < N && col < K) ? B1g[static_cast<size_t>(n) * K + col] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < TK; ++kk) {
      const float a = As[kk][tr];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        acc0[j] = fmaf(a, Bs0[kk][tc + j], acc0[j]);
        if (SWIGLU) acc1[j] = fmaf(a, Bs1[kk][tc + j], acc1[j]);
      }
    }
    __syncthreads();
  }
  const int row = m0 + tr;
  if (row >= rows_g) return;
  float* crow = C + static_cast<size_t>(s_off[g] + row) * N;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int n = n0 + tc + j;
    if (n >= N) continue;
    crow[n] = SWIGLU ? acc0[j] / (1.0f + expf(-acc0[j])) * acc1[j] : acc0[j];
  }
}

template <bool SWIGLU>
cudaError_t launch(const float* A, int64_t a_rows, const int32_t* offsets, int G, int rows_single,
                   const float* B0, const float* B1, int N, int K, float* C,
                   cudaStream_t stream) {
  const int g = offsets ? G : 1;
  const long long rows = offsets ? a_rows : rows_single;
  const long long mt_upper = (rows + TM - 1) / TM + (g > 1 ? g : 0);
  if (mt_upper <= 0) return cudaSuccess;
  const dim3 grid(static_cast<unsigned>(mt_upper), (N + TN - 1) / TN);
  return launch_pdl(grouped_gemm_f32_kernel<SWIGLU>, dim3(grid), dim3(256), 0, stream, A, offsets,
                    G, rows_single, B0, B1, N, K, C);
}

}  // namespace

cudaError_t grouped_swiglu_gateup_f32(const float* A, int64_t a_rows, const int32_t* offsets,
                                      int num_groups, int rows_single, const float* W1,
                                      const float* W3, int F, int K, float* H,
                                      cudaStream_t stream) {
  return launch<true>(A, a_rows, offsets, num_groups, rows_single, W1, W3, F, K, H, stream);
}

cudaError_t grouped_down_f32(const float* A, int64_t a_rows, const int32_t* offsets,
                             int num_groups, int rows_single, const float* W2, int N, int K,
                             float* Y, cudaStream_t stream) {
  return launch<false>(A, a_rows, offsets, num_groups, rows_single, W2, nullptr, N, K, Y, stream);
}

}  // namespace moe
