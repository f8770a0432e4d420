// Launchers of the CUDA kernels behind the C ABI (internal to the library).
#pragma once
#include <cuda_runtime.h>

#include <cstdint>

namespace moe {

// Bits of the device status word kept at the start of the workspace.
constexpr uint32_t kDevBadIndex = 1u;   // expert id outside [0, E) or repeated in a token
constexpr uint32_t kDevTimeout = 2u;    // a bounded wait inside a kernel gave up

// Router ---------------------------------------------------------------------
// Selection-key variants: space 0: key = logit + bias (the default); space 1:
// key = gate score + bias.  noise [T, E] fp32, already scaled by the caller,
// is added to every key when non-null.
struct KeyOpts {
  int space = 0;
  const float* noise = nullptr;
  bool is_default() const { return space == 0 && noise == nullptr; }
};
// logits[T, E] (fp64 scratch) = x . w_router^T (+ logit_offset), exact products
// with fp32 partial sums over 32-wide K chunks added in fp64.
cudaError_t router_logits(bool bf16, const void* x, const void* w_router,
                          const float* logit_offset, int T, int d, int E, double* logits,
                          cudaStream_t stream);
// gate scores, biased selection, top-k, combine weights from the logits.
cudaError_t router_select(const double* logits, const float* sel_bias, int T, int E, int k,
                          int gate, int renorm, const KeyOpts& ko, int32_t* topk_idx,
                          float* topk_w, cudaStream_t stream);

// bf16 router: tensor-core fp32 logits, fast selection with near-tie
// flagging, exact fp64 re-decision of the flagged tokens.  Tokens whose
// top-(k+1) selection keys contain two keys closer than kRefineMargin are
// re-decided on exact logits.  The tensor-core logits are within 5e-6 of the
// exact ones (measured on every logit of the full workloads), so a key gap
// above the margin cannot change order.
constexpr float kRefineMargin = 1e-4f;
// A listed token carries up to kRefineCand candidate experts (the experts
// whose key is within the margin of its (k+1)-th pick); -2 in slot 0 means
// "re-decide over all experts".
constexpr int kRefineCand = 16;
bool router_fused_supported(int E, int k);
cudaError_t router_topk_tc(const void* x, int T, const void* w_router, int E, int K,
                           const float* logit_offset, const float* sel_bias, int k, int gate,
                           int renorm, int32_t* topk_idx, float* topk_w, int32_t* refine_count,
                           int32_t* refine_list, int32_t* refine_cand, uint32_t* status,
                           cudaStream_t stream);
cudaError_t router_logits_tc(const void* x, int T, const void* w_router, int E, int K,
                             float* logits, uint32_t* status, cudaStream_t stream);
cudaError_t router_select_fast(const float* logits, const float* logit_offset,
                               const float* sel_bias, int T, int E, int k, int gate, int renorm,
                               const KeyOpts& ko, int32_t* topk_idx, float* topk_w,
                               int32_t* refine_count, int32_t* refine_list, cudaStream_t stream);
// Exact re-decision of the listed tokens.  refine_cand null: every listed
// token is re-decided over all experts (the unfused path lists no
// candidates; score-space softmax keys need all of them).
cudaError_t router_refine(const void* x, const void* w_router, const float* logit_offset,
                          const float* sel_bias, int T, int d, int E, int k, int gate,
                          int renorm, const KeyOpts& ko, const int32_t* refine_count,
                          const int32_t* refine_list, const int32_t* refine_cand,
                          int32_t* topk_idx, float* topk_w, int sms, cudaStream_t stream);

// logits[t, e] += offset[e]
cudaError_t add_row_offset(float* logits, const float* offset, int T, int E, cudaStream_t stream);

// Router statistics --------------------------------------------------------
int stats_blocks(int T);
// partials: fp64 [stats_blocks(T), 2E+1]; out: float[8] on the device.
cudaError_t router_stats(bool fp64_logits, const void* logits, int T, int E, int gate,
                         const int32_t* topk_idx, int k, double* partials, float* out,
                         cudaStream_t stream);

// Dispatch -------------------------------------------------------------------
constexpr int kRankBlock = 256;   // tokens per histogram block
inline int rank_blocks(int T) { return (T + kRankBlock - 1) / kRankBlock; }
cudaError_t dispatch_rank(const int32_t* topk_idx, int T, int k, int E, int32_t* blk_counts,
                          int32_t* rank_out, uint32_t* status, cudaStream_t stream);
// dispatch_rank followed by dispatch_scan in one launch (the last block to
// finish scans); done: a zeroed counter, zero again when the kernel ends.
// fold_cnt [T, fold_nt] (or null) is set to each token's skipped pairs, the
// starting counts of the combine folded into the down pass.
cudaError_t dispatch_rank_scan(const int32_t* topk_idx, int T, int k, int E, int32_t* blk,
                               int32_t* rank_out, int32_t* counts, int32_t* offsets,
                               uint32_t* status, uint32_t* done, cudaStream_t stream,
                               int32_t* fold_cnt = nullptr, int fold_nt = 0);
cudaError_t dispatch_scan(int32_t* blk_counts, int nblk, int E, int32_t* counts,
                          int32_t* offsets, cudaStream_t stream);
// slot_pos (in: rank inside its block of blk_tokens tokens, out: row) and
// perm_src only, no row copy.  zero (or null): n_zero int32 set to zero,
// the counters of a gate/up launch that copies its own rows.
cudaError_t dispatch_positions(const int32_t* topk_idx, const int32_t* blk_bases,
                               int32_t* slot_pos, int32_t* perm_src, int T, int k, int E,
                               int blk_tokens, cudaStream_t stream, int32_t* zero = nullptr,
                               int n_zero = 0);
cudaError_t dispatch_scatter(bool bf16, const void* x, const int32_t* topk_idx,
                             const int32_t* blk_bases, int32_t* slot_pos, int32_t* perm_src,
                             void* x_perm, int T, int d, int k, int E, int blk_tokens,
                             cudaStream_t stream);

// Experts --------------------------------------------------------------------
// One more group with tensors of its own, run in the same launch after the
// routed groups: the shared expert over all T tokens (A = x or h_sh, B = its
// weights, C = its output).  B1 is the up projection (gate/up pass only).
struct GemmExtraGroup {
  const void* A;
  int rows;
  const void* B0;
  const void* B1;
  int n;     // output columns
  int K;
  void* C;
};
// The routed gate/up launch copies its own A rows (A = x_perm, row r = x
// row perm[r]) while it runs, instead of reading a copy made before it:
// ready [1 + ceil(a_rows / 32)] int32, zero at launch (a unit counter and
// per-32-row block counts).
struct GemmCopy {
  const void* src;       // x [src_rows, K] bf16
  int src_rows;
  const int32_t* perm;   // perm_src [a_rows]
  int32_t* ready;
};
cudaError_t grouped_swiglu_gateup_bf16(const void* A, int64_t a_rows, const int32_t* offsets,
                                       int num_groups, int rows_single, const void* W1,
                                       const void* W3, int F, int K, void* H, uint32_t* status,
                                       cudaStream_t stream,
                                       const GemmExtraGroup* extra = nullptr,
                                       const GemmCopy* copy = nullptr);
cudaError_t grouped_swiglu_gateup_gather_bf16(const void* X, int64_t x_rows, const int32_t* rows,
                                              int64_t R, const int32_t* offsets, int num_groups,
                                              const void* W1, const void* W3, int F, int K,
                                              void* H, uint32_t* status, cudaStream_t stream,
                                              const GemmExtraGroup* extra = nullptr);
// dGU [rows, 2F] = [dH u silu'(g) | dH silu(g)] with g = A W1^T, u = A W3^T
// recomputed on the tensor cores (groups as for the gate/up pass).
cudaError_t grouped_swiglu_bwd_bf16(const void* A, int64_t a_rows, const int32_t* offsets,
                                    int num_groups, int rows_single, const void* W1,
                                    const void* W3, int F, int K, const void* dH, void* dGU,
                                    uint32_t* status, cudaStream_t stream);
// The combine folded into the down pass (see GemmArgs in
// grouped_gemm_sm100.cu): counts [T, nt] set by dispatch_rank_scan, nt =
// ceil(N / down_tile_cols(N, K)); out [T, N] receives the combined rows.
struct GemmFold {
  int32_t* cnt;
  int nt, T, k;
  const int32_t* src;    // perm_src [T k]
  const int32_t* slot;   // slot_pos [T, k]
  const float* w;        // topk_w [T, k]
  void* out;
};
int down_tile_cols(int N, int K);
cudaError_t grouped_down_bf16(const void* A, int64_t a_rows, const int32_t* offsets,
                              int num_groups, int rows_single, const void* W2, int N, int K,
                              void* Y, uint32_t* status, cudaStream_t stream,
                              const GemmExtraGroup* extra = nullptr,
                              const GemmFold* fold = nullptr);
// Y[r] = A[r] B_g, B_g [K, N] read MN-major (no transposed copy): its first
// b0_rows rows from B0 [G * b0_rows, N], the others from B1.
cudaError_t grouped_gemm_bmn_bf16(const void* A, int64_t a_rows, const int32_t* offsets,
                                  int num_groups, int rows_single, const void* B0,
                                  const void* B1, int b0_rows, int N, int K, void* Y,
                                  uint32_t* status, cudaStream_t stream);
// fp32 output variant, all K rows from B0 (group g: rows [g K, g K + K),
// rows at or past b0_total_rows read as zero).
cudaError_t grouped_gemm_bmn_f32out(const void* A, int64_t a_rows, const int32_t* offsets,
                                    int num_groups, int rows_single, const void* B0,
                                    int b0_rows, int64_t b0_total_rows, int N, float* Y,
                                    uint32_t* status, cudaStream_t stream);
cudaError_t grouped_swiglu_gateup_f32(const float* A, int64_t a_rows, const int32_t* offsets,
                                      int num_groups, int rows_single, const float* W1,
                                      const float* W3, int F, int K, float* H,
                                      cudaStream_t stream);
cudaError_t grouped_down_f32(const float* A, int64_t a_rows, const int32_t* offsets,
                             int num_groups, int rows_single, const float* W2, int N, int K,
                             float* Y, cudaStream_t stream);

// Backward -------------------------------------------------------------------
// K-grouped weight gradient C_g [M, N] = A_g^T B_g over the rows
// [offsets[g], offsets[g+1]) (offsets null: one group of `rows` rows) of
// A [rows, lda] (columns a_col0 ..) and B [rows, ldb] (columns b_col0 ..),
// both read MN-major; C [G, M, N] bf16.
cudaError_t grouped_wgrad_bf16(const void* A, int lda, int a_col0, const void* B, int ldb,
                               int b_col0, int64_t rows, const int32_t* offsets, int G, int M,
                               int N, void* C, uint32_t* status, cudaStream_t stream);
cudaError_t bwd_dy(const void* dout, const void* y_perm, const int32_t* slot_pos,
                   const float* topk_w, void* dy, float* dw, int T, int d, int k,
                   cudaStream_t stream);
cudaError_t dx_gather(const void* dxp, const int32_t* slot_pos, const float* dxr, const void* dxs,
                      void* dx, int T, int d, int k, cudaStream_t stream);
cudaError_t router_dlogits(const float* logits, const float* offset, const int32_t* topk_idx,
                           const float* topk_w, const float* dw, int T, int E, int k, int gate,
                           int renorm, float* dlogits, cudaStream_t stream);
// x_perm[r] = x[perm_src[r]] for r < R when *flag is non-zero (a forward
// that gathered its rows); nothing otherwise.  bf16 rows of d elements.
cudaError_t fill_xperm(const void* x, const int32_t* perm_src, const uint32_t* flag,
                       void* x_perm, long long R, int T, int d, cudaStream_t stream);
// Router gradients on the tensor cores: dlogits split into three bf16 terms
// (exact), Ep = E rounded up to 64, G token slices of Ks tokens for dW.
struct RouterGradShape {
  int Ep, Ks, G;
};
RouterGradShape router_grad_shape(int T, int E);
// adx [T, 3 Ep] and adw [G, 3 Ep, Ks] bf16, goff [G + 1] = g * 3 Ep.
cudaError_t router_grad_split(const float* dlogits, int T, int E, const RouterGradShape& r,
                              void* adx, void* adw, int32_t* goff, cudaStream_t stream);
// out [E, d] fp32 = sum over slices and terms of part [G, 3 Ep, d].
cudaError_t router_grad_reduce(const float* part, const RouterGradShape& r, int E, int d,
                               float* out, cudaStream_t stream);

// Combine / bias ---------------------------------------------------------------
cudaError_t combine(bool bf16, const void* y_perm, const int32_t* slot_pos, const float* topk_w,
                    const void* y_shared, void* out, int T, int d, int k, cudaStream_t stream);
cudaError_t bias_update(const int32_t* counts, float* bias, int E, float target, float thresh,
                        float starved_add, float rate, float clamp, cudaStream_t stream);
cudaError_t bias_update_sign(const int32_t* counts, float* bias, int E, float rate,
                             cudaStream_t stream);

}  // namespace moe
