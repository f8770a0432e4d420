/*
 * moe.h -- C ABI of libmoe_b200.so: the forward pass of a Mixture-of-Experts
 * FFN layer on NVIDIA B200 (sm_100a).
 *
 * The layer (sources by page title and section):
 *   router    logits = x . Wr^T in fp32, scores = sigmoid(logits) or softmax
 *             over all experts, selection keys = logits + sel_bias, top-k of
 *             the keys, combine weights = the unbiased scores of the chosen
 *             experts, optionally divided by (their sum + 1e-9).
 *             ("moe-200m-qwen3-100b" README, "SigmoidRouter"; SpecForge PR
 *             #930, "What this adds": qwen3 preset, softmax + norm_topk_prob.)
 *   experts   E routed SwiGLU experts  y = W2 (silu(W1 x) * (W3 x)), weights
 *             stacked [E, out, in] (SpecForge PR #930, "Why FSDP is enough
 *             here"; per-expert keys w1/w2/w3 in SpecForge PR #931, "What
 *             works"), plus optionally one always-on shared SwiGLU expert.
 *   combine   out = shared(x) + sum_j w_j * expert_{idx_j}(x)
 *             ("moe-200m-qwen3-100b" README, "Architecture diagram").
 *   bias      aux-loss-free controller from per-expert counts
 *             ("moe-200m-qwen3-100b" README, "SigmoidRouter", step_bias_update).
 *
 * Conventions shared by every call:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library
 *     never allocates or frees device memory.  Scratch comes from the caller's
 *     workspace `ws` of `ws_bytes` bytes (>= moe_workspace_size(cfg)), 256-byte
 *     aligned -- except for moe_permute_noalloc, whose scratch is a fixed
 *     array in the library's own device memory (see there).  Tensors are
 *     dense row-major.  "act" below means the activation / weight dtype
 *     cfg->dtype (fp32 or bf16); router logits, scores, weights and the
 *     selection bias are fp32 whatever the act dtype.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call is
 *     asynchronous on it and performs no host synchronisation, except
 *     moe_device_status().
 *   - Arguments are validated before anything is launched; on error nothing
 *     is launched and an error code is returned.  T == 0 is a valid no-op.
 *   - Problems only the device can see (an expert id outside [0, E) in a
 *     caller-supplied topk_idx; a bounded wait inside a kernel that gave up)
 *     never fault: the kernel records them in a status word inside `ws` and
 *     skips the offending work.  Each call clears the word when it starts;
 *     read it with moe_device_status().
 *   - No global state (except moe_permute_noalloc's fixed scratch array and
 *     its per-device address cache), no exceptions.  Calls on different
 *     streams with different workspaces may run concurrently.
 *   - Limits: 1 <= top_k <= min(E, 32), E <= 256.  bf16: d_model, d_ff and
 *     d_ff_shared multiples of 128; fp32: d_model multiple of 4.  Pointers
 *     16-byte aligned.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID = 1,      /* bad argument: null pointer, size, alignment     */
  MOE_ERR_UNSUPPORTED = 2,  /* valid layer, but outside this build's limits    */
  MOE_ERR_WORKSPACE = 3,    /* ws_bytes < moe_workspace_size(cfg)               */
  MOE_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed             */
  MOE_ERR_TIMEOUT = 5,      /* device status: a bounded wait gave up            */
  MOE_ERR_DATA = 6          /* device status: expert id outside [0, E) skipped  */
} moe_status;

typedef enum { MOE_GATE_SOFTMAX = 0, MOE_GATE_SIGMOID = 1 } moe_gate;
typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

/* Shape and recipe of one MoE layer (MoEModelConfig fields of the
 * "moe-200m-qwen3-100b" README, plus the qwen3 preset switches of SpecForge
 * PR #930).  Plain int32 fields so the layout is the same from every language. */
typedef struct {
  int32_t T;               /* tokens in the batch                          */
  int32_t d_model;         /* hidden size d                                */
  int32_t n_experts;       /* routed experts E                             */
  int32_t d_ff;            /* routed expert width F                        */
  int32_t top_k;           /* experts per token k                          */
  int32_t n_shared;        /* 0 or 1 always-on shared expert               */
  int32_t d_ff_shared;     /* shared expert width (0 when n_shared == 0)   */
  int32_t gate;            /* moe_gate                                     */
  int32_t norm_topk_prob;  /* 1: w /= (sum_j w_j + 1e-9)                   */
  int32_t dtype;           /* moe_dtype of x, weights, out and the
                              intermediate activations                     */
} moe_config;

/* Expert weights, stacked [E, out, in] (SpecForge PR #930):
 *   w1 [E, F, d] gate, w3 [E, F, d] up, w2 [E, d, F] down;
 *   ws1 [Fs, d], ws3 [Fs, d], ws2 [d, Fs] for the shared expert (NULL when
 *   n_shared == 0).  All act dtype. */
typedef struct {
  const void* w1;
  const void* w3;
  const void* w2;
  const void* ws1;
  const void* ws3;
  const void* ws2;
} moe_expert_weights;

/* Gradients of the expert weights: the same shapes and dtype as the
 * weights in moe_expert_weights; dws* are NULL when n_shared == 0. */
typedef struct {
  void* dw1;
  void* dw3;
  void* dw2;
  void* dws1;
  void* dws3;
  void* dws2;
} moe_expert_grads;

/* Bytes of workspace every call below needs for this configuration
 * (0 on an invalid configuration). */
size_t moe_workspace_size(const moe_config* cfg);

/* Validate a configuration without launching anything. */
moe_status moe_check_config(const moe_config* cfg);

/* Router: logits, gate, biased selection, top-k and combine weights.
 * ("moe-200m-qwen3-100b" README, "SigmoidRouter" forward; "Per-layer
 * numerics": routing in fp32.  SpecForge PR #930 "What this adds".)
 *   x [T, d] act;  w_router [E, d] act;  sel_bias [E] fp32 or NULL (moves the
 *   selection only, never the weights); logit_offset [E] fp32 or NULL (a
 *   per-expert constant added to the logits before the gate and the
 *   selection).
 *   out: topk_idx [T, k] int32, descending selection key, equal keys -> lower
 *   expert id; topk_w [T, k] fp32.
 *   bf16 layers: logits from exact bf16 products on the tensor cores, summed
 *   in fp32 per 128-wide K chunk with the chunk sums added in fp32 (within
 *   5e-6 of the exact logits); keys, gate and weights in fp32; every token
 *   with two of its top-(k+1) keys closer than 1e-4 is re-decided on exact
 *   logits (fp64 sums) over its candidate experts, so the selection equals
 *   the one taken on exact logits.
 *   fp32 layers: products in fp32 summed in fp32 over 32-wide K chunks, chunk
 *   sums added in fp64; keys, gate and renormalisation in fp64.  Weights are
 *   stored as fp32 in both cases. */
moe_status moe_router_topk(const moe_config* cfg, const void* x, const void* w_router,
                           const float* sel_bias, const float* logit_offset,
                           int32_t* topk_idx, float* topk_w,
                           void* ws, size_t ws_bytes, void* stream);

/* Selection-key variants of the router.
 *   bias_space 0: key = logit + sel_bias (SigmoidRouter.forward of the
 *     "moe-200m-qwen3-100b" README; what moe_router_topk does).
 *   bias_space 1: key = gate score + sel_bias, the score being sigmoid(logit)
 *     or the softmax probability over all E experts (the score-space
 *     placement of the "noaux_tc" balance bias named on the page-3 model
 *     card, which prints no code for it).
 *   sel_noise: NULL, or [T, E] fp32 on the device, added to every key: the
 *     training-time exploration noise of SigmoidRouter.forward
 *     (sel_logits += randn * noise_std), drawn and scaled by the caller
 *     (noise_std * standard-normal draws), so the library draws nothing.
 * The noise and the bias move the selection only; the weights are the
 * unbiased gate scores of the chosen experts, as in moe_router_topk. */
typedef struct {
  int32_t bias_space;        /* 0 or 1                                  */
  int32_t reserved;          /* 0                                       */
  const float* sel_noise;    /* [T, E] fp32 or NULL                     */
} moe_router_opts;

/* moe_router_topk with the key variants above (arguments and outputs as
 * there; opts must not be NULL; bias_space outside {0, 1} or an unaligned
 * sel_noise is MOE_ERR_INVALID).  Runs the unfused tensor-core path for
 * bf16 layers: fp32 logits, fp32 keys, exact fp64 re-decision over all
 * experts of every token with two of its top-(k+1) keys closer than 1e-4.
 * With bias_space 0 and no noise it returns what moe_router_topk returns. */
moe_status moe_router_topk_opts(const moe_config* cfg, const void* x, const void* w_router,
                                const float* sel_bias, const float* logit_offset,
                                const moe_router_opts* opts, int32_t* topk_idx, float* topk_w,
                                void* ws, size_t ws_bytes, void* stream);

/* Router GEMM alone: logits [T, E] fp32 = x . w_router^T (+ logit_offset),
 * for bf16 layers (fp32 layers return MOE_ERR_UNSUPPORTED).  Tensor cores,
 * exact bf16 products, fp32 accumulation: these are the logits moe_router_topk
 * selects from before it re-decides near ties on exact logits. */
moe_status moe_router_logits(const moe_config* cfg, const void* x, const void* w_router,
                             const float* logit_offset, float* logits,
                             void* ws, size_t ws_bytes, void* stream);

/* Router losses and health metrics for a batch and its routing (the aux
 * dict of SigmoidRouter.forward, "moe-200m-qwen3-100b" README; load metrics
 * of SpecForge PR #931, "What to watch").  Recomputes the logits
 * (tensor cores for bf16) and reads topk_idx [T, k] (e.g. from
 * moe_router_topk).  stats: 8 floats on the device:
 *   [0] z_loss = mean_t logsumexp_e(logits)^2
 *   [1] aux_loss = E * sum_e (fraction of tokens choosing e) * (mean score of e)
 *   [2] cv = std(counts, Bessel) / max(mean(counts), 1)   (NaN for E = 1)
 *   [3] entropy of the normalised mean scores, in bits
 *   [4] load_max_ratio = max(counts) / mean(counts)   (ceiling E / k)
 *   [5] fraction of experts with no tokens;  [6], [7] = 0.
 * Deterministic (fixed reduction order). */
moe_status moe_router_stats(const moe_config* cfg, const void* x, const void* w_router,
                            const float* logit_offset, const int32_t* topk_idx, float* stats,
                            void* ws, size_t ws_bytes, void* stream);

/* Dispatch: per-expert counts, offsets, and the stable expert-contiguous
 * permutation of the T*k routed rows, with x gathered into that order.
 * (Grouped-GEMM dispatch, SpecForge PR #930 "Why FSDP is enough here" and
 * PR #931 "What works": grouped GEMM checked against a sorted loop.)
 *   topk_idx [T, k] int32 (a pair whose id is outside [0, E) or repeats an
 *   id earlier in the same token is skipped and reported as MOE_ERR_DATA by
 *   moe_device_status); x [T, d] act.
 *   out: counts [E] int32; offsets [E+1] int32 (exclusive prefix of counts);
 *   slot_pos [T, k] int32 = row of pair (t, j) in the permuted order, i.e. the
 *   position of (expert, t) in the stable sort of all pairs by (expert, token)
 *   (-1 for a skipped pair); perm_src [T*k] int32 = token of each row;
 *   x_perm [T*k, d] act, x_perm[slot_pos[t, j]] = x[t]. */
moe_status moe_permute(const moe_config* cfg, const int32_t* topk_idx, const void* x,
                       int32_t* counts, int32_t* offsets, int32_t* slot_pos,
                       int32_t* perm_src, void* x_perm,
                       void* ws, size_t ws_bytes, void* stream);

/* Experts: grouped SwiGLU over the expert segments of x_perm, and the shared
 * expert over x.  ("moe-200m-qwen3-100b" README, "Architecture diagram":
 * routed SwiGLU experts and one always-on shared expert.)
 *   x_perm [T*k, d] act; offsets [E+1] int32 (rows of expert e are
 *   offsets[e] .. offsets[e+1]-1, offsets[E] <= T*k); weights as above;
 *   x [T, d] act (read only when n_shared == 1).
 *   out: y_perm [T*k, d] act, row r = expert_e(x_perm[r]) for the e owning r
 *   (rows at or past offsets[E] are left untouched); y_shared [T, d] act or
 *   NULL when n_shared == 0.  bf16: fp32 accumulation, the SwiGLU product
 *   h = silu(g) * u is rounded to bf16 before the down projection. */
moe_status moe_grouped_swiglu(const moe_config* cfg, const void* x_perm, const int32_t* offsets,
                              const moe_expert_weights* w, const void* x,
                              void* y_perm, void* y_shared,
                              void* ws, size_t ws_bytes, void* stream);

/* Combine: out[t] = y_shared[t] + sum_{j<k, j ascending} topk_w[t, j] *
 * y_perm[slot_pos[t, j]], accumulated in fp32, stored once in act dtype.
 * ("moe-200m-qwen3-100b" README, "Architecture diagram": weighted sum.)
 *   y_shared may be NULL (no shared expert).  A slot_pos entry outside
 *   [0, T*k) is skipped (contributes nothing); this call has no workspace, so
 *   such entries are not reported. */
moe_status moe_combine(const moe_config* cfg, const void* y_perm, const int32_t* slot_pos,
                       const float* topk_w, const void* y_shared, void* out, void* stream);

/* Selection-bias update from per-expert counts, in place, fp32, in the
 * order of step_bias_update ("moe-200m-qwen3-100b" README, "SigmoidRouter"):
 *   p = c / max(sum c, 1);  err = fp32(1/E) - p;
 *   err += fp32(starved_add) where p < fp32(starved_frac * (1/E));
 *   bias = clamp(bias + err * fp32(rate), -fp32(clamp), +fp32(clamp)).
 * Each step is one correctly rounded fp32 operation (no fused multiply-add).
 * counts must already be summed over data-parallel ranks (the README's
 * all-reduce before the update).  Defaults on the page: rate 1e-3,
 * starved_frac 0.1, starved_add 0.5, clamp 10. */
moe_status moe_bias_update(const moe_config* cfg, const int32_t* counts, float* sel_bias,
                           double rate, double starved_frac, double starved_add,
                           double clamp, void* stream);

/* Selection-bias update of the noaux_tc kind: one fixed step per call
 * (micro-batch) toward balance, fp32, in place, no clamp:
 *   bias_e += fp32(rate) * sign(fp32(sum c) / E - c_e)      (sign(0) = 0).
 * SpecForge PR #931, "What to watch": at rate 0.001 and 64 accumulation
 * steps a starved expert's bias grows 0.064 per optimizer step. */
moe_status moe_bias_update_sign(const moe_config* cfg, const int32_t* counts, float* sel_bias,
                                double rate, void* stream);

/* The whole layer forward: router, dispatch, grouped SwiGLU experts (+ shared
 * expert), combine.  Inputs as above; out [T, d] act.  Also returns the
 * routing (topk_idx [T, k], topk_w [T, k]) and counts [E] for the caller's
 * bias update; intermediates live in ws. */
moe_status moe_forward(const moe_config* cfg, const void* x, const void* w_router,
                       const float* sel_bias, const float* logit_offset,
                       const moe_expert_weights* w, void* out,
                       int32_t* topk_idx, float* topk_w, int32_t* counts,
                       void* ws, size_t ws_bytes, void* stream);

/* Alternatives of moe_forward's expert path, chosen per call.
 *   gather_rows 0 (default): dispatch writes the permuted copy x_perm and the
 *     gate/up grouped GEMM reads it with TMA tiles.
 *   gather_rows 1 (bf16 layers only): dispatch writes no x_perm; the gate/up
 *     GEMM gathers each tile's rows from x through the permutation (TMA
 *     tile::gather4 loads, four rows per load).  Same results.
 *   fold_combine 0 (default): a separate combine launch reads y_perm (and
 *     the shared expert's rows) and writes out.
 *   fold_combine 1 (bf16 layers only): the down GEMM forms out itself: after
 *     a warp stores its 32 rows of an output tile it counts them per token,
 *     and the warp that completes a token's column tile (its k routed rows
 *     and the shared row) sums them into out in the combine's order.  Same
 *     results; one launch fewer, but measured slower on B200 (the summing
 *     warps hold the down GEMM's epilogue).  Combinable with gather_rows.
 *   scatter_in_gemm 1 (bf16 layers only; not with gather_rows): dispatch
 *     writes only the rows' positions, and the gate/up GEMM launch fills
 *     x_perm itself while it runs: two extra warps per CTA copy x's rows in
 *     row order and count them per 32-row block, and each tile's loads wait
 *     (bounded) for the blocks of its rows.  Same results; x_perm is kept
 *     for moe_backward as with the default.
 *   reserved: must be 0. */
typedef struct {
  int32_t gather_rows;
  int32_t fold_combine;
  int32_t scatter_in_gemm;
  int32_t reserved[1];
} moe_forward_opts;

/* moe_forward with the options above (opts must not be NULL; a field
 * outside its values, or gather_rows with scatter_in_gemm, is
 * MOE_ERR_INVALID; any of the three on an fp32 layer is
 * MOE_ERR_UNSUPPORTED). */
moe_status moe_forward_ex(const moe_config* cfg, const void* x, const void* w_router,
                          const float* sel_bias, const float* logit_offset,
                          const moe_expert_weights* w, void* out,
                          int32_t* topk_idx, float* topk_w, int32_t* counts,
                          const moe_forward_opts* opts, void* ws, size_t ws_bytes,
                          void* stream);

/* Where moe_forward keeps the routed order inside its workspace (host
 * arithmetic only, nothing is launched or read): offsets [E+1], slot_pos
 * [T, k] and perm_src [T*k] int32, as moe_permute defines them, valid after a
 * moe_forward / moe_forward_ex call on `ws` has completed on its stream and
 * until the next call that uses `ws`.  The pointers point into ws; the
 * caller reads them (e.g. to check the permutation, or for its own backward)
 * and must not write them while moe_backward may still read them. */
moe_status moe_forward_dispatch_view(const moe_config* cfg, const void* ws, size_t ws_bytes,
                                     const int32_t** offsets, const int32_t** slot_pos,
                                     const int32_t** perm_src);

/* moe_forward with CUDA events (cudaEvent_t, created by the caller) recorded
 * on `stream` at the phase boundaries, for per-phase device timing:
 *   events[0] start            events[1] after the router
 *   events[2] after dispatch   events[3] after the gate/up GEMM
 *   events[4] after the down GEMM
 *   events[5] right after events[4] (the shared expert runs as one more
 *             group inside the two GEMM launches of bf16 layers)
 *   events[6] after the combine (end)
 * Same launches and results as moe_forward. */
#define MOE_FORWARD_PHASES 6
moe_status moe_forward_profiled(const moe_config* cfg, const void* x, const void* w_router,
                                const float* sel_bias, const float* logit_offset,
                                const moe_expert_weights* w, void* out,
                                int32_t* topk_idx, float* topk_w, int32_t* counts,
                                void* ws, size_t ws_bytes, void* stream,
                                void* const* events);

/* moe_permute without a workspace, for callers that cannot allocate device
 * memory: a host program that links only this library and has no device
 * allocator, or a serving loop on a fixed memory plan that must not call
 * cudaMalloc/cudaFree once running (they synchronise the device and can fail
 * when memory is fragmented).  The pages have no counterpart; this is a
 * deployment variant of the dispatch call above, with the same arguments
 * minus ws/ws_bytes and the same outputs.
 *   Scratch: a fixed array of MOE_PERMUTE_NOALLOC_MAX_BLOCK_COUNTS int32 block
 *   counts (+256 B for a status word) in the library's own device memory,
 *   one copy per GPU that loads the library, held until the process exits.
 *   Limit: ceil(T/256) * E <= MOE_PERMUTE_NOALLOC_MAX_BLOCK_COUNTS (e.g.
 *   T <= 524288 at E = 128); larger calls return MOE_ERR_WORKSPACE without
 *   launching anything.
 *   The first call on a device looks up that device's copy of the array
 *   (cudaGetSymbolAddress, with the device current); make that first call
 *   before any stream capture.  The call allocates nothing.
 *   Every call shares the one array and leaves its contents behind; calls
 *   whose work overlaps on the GPU (other streams, other threads) race on it
 *   and must be serialised by the caller.  Pairs with an invalid or repeated
 *   expert id are skipped (slot_pos -1, offsets[E] < T*k); there is no
 *   workspace, so moe_device_status cannot report them. */
#define MOE_PERMUTE_NOALLOC_MAX_BLOCK_COUNTS 262144
moe_status moe_permute_noalloc(const moe_config* cfg, const int32_t* topk_idx, const void* x,
                               int32_t* counts, int32_t* offsets, int32_t* slot_pos,
                               int32_t* perm_src, void* x_perm, void* stream);

/* Synchronise `stream`, read and clear the device status word in ws.
 * Returns MOE_OK, MOE_ERR_DATA, MOE_ERR_TIMEOUT or MOE_ERR_CUDA; the raw
 * flag bits are stored in *flags when flags is not NULL. */
moe_status moe_device_status(void* ws, size_t ws_bytes, void* stream, uint32_t* flags);

/* Synchronise `stream` and store in *count how many tokens the last bf16
 * router call of this workspace re-decided on exact logits (tokens whose
 * top-(k+1) selection keys held two keys closer than the router's margin).
 * Diagnostic only; 0 for fp32 layers. */
moe_status moe_router_refined_tokens(void* ws, size_t ws_bytes, void* stream, int32_t* count);

/* Diagnostic: launch a kernel that waits on a barrier phase nothing
 * completes, using the same bounded wait as the tensor-core kernels, with a
 * limit of limit_seconds (0 < limit <= 2).  The wait gives up, the kernel
 * records the timeout in the status word of ws (>= 256 bytes, 256-byte
 * aligned) and returns; moe_device_status then reports MOE_ERR_TIMEOUT and
 * the context stays usable.  Has no counterpart on the pages. */
moe_status moe_selftest_bounded_wait(void* ws, size_t ws_bytes, double limit_seconds,
                                     void* stream);

/* Static description of a status code. */
const char* moe_status_string(moe_status s);

/* Backward of the layer (bf16 layers; fp32 layers return
 * MOE_ERR_UNSUPPORTED).  The pages train the layer (the "moe-200m-qwen3-100b"
 * README trains SigmoidRouter models end to end; SpecForge PR #930 trains the
 * qwen3 drafter); this is the gradient of <dout, out> for the forward above:
 *   combine   dw[t, j] = <dout[t], y[t, j]>, expert output gradient w[t, j] dout[t],
 *             shared expert output gradient dout[t];
 *   experts   SwiGLU chain rule, silu'(g) = s(g) (1 + g (1 - s(g)));
 *   router    no gradient through the selection (bias, noise); through the
 *             weights w = s_picked / (sum + 1e-9) (or s_picked) with s the
 *             sigmoid or the softmax over all E: dlogits, then
 *             dw_router = dlogits^T x and dx += dlogits w_router (fp32).
 * Inputs: the forward's x, w_router, logit_offset, weights, topk_idx,
 * topk_w (as moe_forward returned them) and dout [T, d] act.  fws is the
 * workspace of that moe_forward (or moe_forward_ex) call, unchanged since
 * (the backward reads the routed order and the saved activations h and y
 * from it, and x_perm unless that forward gathered its rows).  bws:
 * backward scratch of moe_backward_workspace_size(cfg) bytes,
 * 256-byte aligned; its first word is a device status word read with
 * moe_device_status(bws, ...).
 * Outputs: dx [T, d] act; dw_router [E, d] fp32; g->dw1, dw3 [E, F, d],
 * dw2 [E, d, F] act (and the shared expert's).  Activation gradients are
 * bf16 between the steps, the contractions accumulate in fp32 on the tensor
 * cores.  The router's dlogits stay fp32: its two products run with dlogits
 * written as three bf16 terms whose sum is the fp32 value to within fp32
 * rounding, so every product with the bf16 x or w_router is exact and the
 * fp32 accumulation is the only rounding. */
size_t moe_backward_workspace_size(const moe_config* cfg);
moe_status moe_backward(const moe_config* cfg, const void* x, const void* w_router,
                        const float* logit_offset, const moe_expert_weights* w,
                        const int32_t* topk_idx, const float* topk_w, const void* dout, void* dx,
                        float* dw_router, const moe_expert_grads* g, void* fws, size_t fws_bytes,
                        void* bws, size_t bws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
