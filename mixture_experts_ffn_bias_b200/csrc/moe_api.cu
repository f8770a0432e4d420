// C ABI of the MoE FFN layer (declared in include/moe.h): argument
// validation, workspace layout and the launch sequence of each call.
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "../../include/moe.h"
#include "kernels.h"

namespace {

constexpr size_t kAlign = 256;
inline size_t up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

// Workspace layout shared by every call.  Byte offsets from the base.
struct Layout {
  size_t status, blk, offsets, slot_pos, perm_src, refine, refine_cand, stats, logits, x_perm, h,
      y_perm, h_sh, y_sh, fold, copy_ready, total;
};

inline size_t esize(const moe_config& c) { return c.dtype == MOE_BF16 ? 2 : 4; }

Layout layout(const moe_config& c) {
  const size_t T = static_cast<size_t>(c.T), d = c.d_model, E = c.n_experts, F = c.d_ff,
               k = c.top_k, R = T * k, es = esize(c);
  const size_t Fs = c.n_shared ? static_cast<size_t>(c.d_ff_shared) : 0;
  Layout L{};
  size_t o = 0;
  // status area: four words (see clear_status)
  L.status = o;   o += up(4 * sizeof(uint32_t));
  L.blk = o;      o += up(static_cast<size_t>(moe::rank_blocks(c.T)) * E * 4);
  L.offsets = o;  o += up((E + 1) * 4);
  L.slot_pos = o; o += up(R * 4);
  L.perm_src = o; o += up(R * 4);
  L.refine = o;   o += up(T * 4);
  L.refine_cand = o; o += up(T * moe::kRefineCand * 4);
  L.stats = o;    o += up(static_cast<size_t>(moe::stats_blocks(c.T)) * (2 * E + 1) * 8);
  L.logits = o;   o += up(T * E * 8);
  L.x_perm = o;   o += up(R * d * es);
  L.h = o;        o += up(R * F * es);
  L.y_perm = o;   o += up(R * d * es);
  L.h_sh = o;     o += up(T * Fs * es);
  L.y_sh = o;     o += up(c.n_shared ? T * d * es : 0);
  // the folded combine's counts: [T, column tiles of the down GEMM], at
  // most d / 128 tiles (bf16 only)
  L.fold = o;     o += up(c.dtype == MOE_BF16 ? T * ((d + 127) / 128) * 4 : 0);
  // the counters of a gate/up launch that copies its own rows (bf16 only)
  L.copy_ready = o; o += up(c.dtype == MOE_BF16 ? (1 + (R + 31) / 32) * 4 : 0);
  L.total = o;
  return L;
}

template <typename P>
inline P* at(void* ws, size_t off) {
  return reinterpret_cast<P*>(static_cast<uint8_t*>(ws) + off);
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

moe_status check_cfg(const moe_config* c) {
  if (c == nullptr) return MOE_ERR_INVALID;
  if (c->T < 0 || c->d_model < 1 || c->n_experts < 1 || c->d_ff < 1 || c->top_k < 1)
    return MOE_ERR_INVALID;
  if (c->top_k > c->n_experts) return MOE_ERR_INVALID;
  if (c->n_shared != 0 && c->n_shared != 1) return MOE_ERR_INVALID;
  if (c->n_shared == 1 && c->d_ff_shared < 1) return MOE_ERR_INVALID;
  if (c->gate != MOE_GATE_SOFTMAX && c->gate != MOE_GATE_SIGMOID) return MOE_ERR_INVALID;
  if (c->norm_topk_prob != 0 && c->norm_topk_prob != 1) return MOE_ERR_INVALID;
  if (c->dtype != MOE_F32 && c->dtype != MOE_BF16) return MOE_ERR_INVALID;
  if (c->n_experts > 256 || c->top_k > 32) return MOE_ERR_UNSUPPORTED;
  if (static_cast<long long>(c->T) * c->top_k > 0x3fffffffLL) return MOE_ERR_UNSUPPORTED;
  if (c->dtype == MOE_BF16) {
    if (c->d_model % 128 || c->d_ff % 128 || (c->n_shared && c->d_ff_shared % 128))
      return MOE_ERR_UNSUPPORTED;
  } else {
    if (c->d_model % 4) return MOE_ERR_UNSUPPORTED;
  }
  return MOE_OK;
}

moe_status check_ws(const moe_config* c, const void* ws, size_t ws_bytes) {
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1))) return MOE_ERR_INVALID;
  if (ws_bytes < layout(*c).total) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

inline cudaStream_t S(void* s) { return static_cast<cudaStream_t>(s); }

#define MOE_TRY(expr)                                   \
  do {                                                  \
    if ((expr) != cudaSuccess) return MOE_ERR_CUDA;     \
  } while (0)

// Word 0: device status flags; word 1: number of tokens the router listed
// for exact re-decision; word 2: non-zero when the last forward kept no
// permuted copy of x (gathered gate/up rows); word 3: the rank kernel's
// count of finished blocks.
moe_status clear_status(void* ws, cudaStream_t s) {
  MOE_TRY(cudaMemsetAsync(at<uint32_t>(ws, 0), 0, 4 * sizeof(uint32_t), s));
  return MOE_OK;
}

int device_sms() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// Router into caller buffers; logits scratch in ws.
moe_status run_router(const moe_config* c, const void* x, const void* w_router,
                      const float* sel_bias, const float* logit_offset, int32_t* topk_idx,
                      float* topk_w, void* ws, cudaStream_t s,
                      const moe::KeyOpts& ko = moe::KeyOpts{}) {
  const Layout L = layout(*c);
  if (c->dtype == MOE_BF16) {
    float* logits = at<float>(ws, L.logits);
    int32_t* count = at<int32_t>(ws, L.status) + 1;
    int32_t* list = at<int32_t>(ws, L.refine);
    // the key variants take the unfused path: fp32 logits, a select kernel
    // and exact re-decision over all experts
    const bool fused = ko.is_default() && moe::router_fused_supported(c->n_experts, c->top_k);
    int32_t* cand = at<int32_t>(ws, L.refine_cand);
    if (fused) {
      MOE_TRY(moe::router_topk_tc(x, c->T, w_router, c->n_experts, c->d_model, logit_offset,
                                  sel_bias, c->top_k, c->gate, c->norm_topk_prob, topk_idx,
                                  topk_w, count, list, cand, at<uint32_t>(ws, L.status), s));
    } else {
      MOE_TRY(moe::router_logits_tc(x, c->T, w_router, c->n_experts, c->d_model, logits,
                                    at<uint32_t>(ws, L.status), s));
      MOE_TRY(moe::router_select_fast(logits, logit_offset, sel_bias, c->T, c->n_experts,
                                      c->top_k, c->gate, c->norm_topk_prob, ko, topk_idx, topk_w,
                                      count, list, s));
    }
    MOE_TRY(moe::router_refine(x, w_router, logit_offset, sel_bias, c->T, c->d_model,
                               c->n_experts, c->top_k, c->gate, c->norm_topk_prob, ko, count,
                               list, fused ? cand : nullptr, topk_idx, topk_w, device_sms(), s));
    return MOE_OK;
  }
  double* logits = at<double>(ws, L.logits);
  MOE_TRY(moe::router_logits(false, x, w_router, logit_offset, c->T, c->d_model, c->n_experts,
                             logits, s));
  MOE_TRY(moe::router_select(logits, sel_bias, c->T, c->n_experts, c->top_k, c->gate,
                             c->norm_topk_prob, ko, topk_idx, topk_w, s));
  return MOE_OK;
}

// fold_nt > 0: also set the folded combine's counts ([T, fold_nt] in ws).
// copy_counters (x_perm == nullptr only): also zero the counters of a gate/up
// launch that copies its own rows.
moe_status run_permute(const moe_config* c, const int32_t* topk_idx, const void* x,
                       int32_t* counts, int32_t* offsets, int32_t* slot_pos, int32_t* perm_src,
                       void* x_perm, void* ws, cudaStream_t s, int fold_nt = 0,
                       bool copy_counters = false) {
  const Layout L = layout(*c);
  int32_t* blk = at<int32_t>(ws, L.blk);
  uint32_t* status = at<uint32_t>(ws, L.status);
  MOE_TRY(moe::dispatch_rank_scan(topk_idx, c->T, c->top_k, c->n_experts, blk, slot_pos, counts,
                                  offsets, status, status + 3, s,
                                  fold_nt > 0 ? at<int32_t>(ws, L.fold) : nullptr, fold_nt));
  if (x_perm == nullptr) {   // rows only; the experts gather x through perm_src
    const int n_zero =
        copy_counters ? 1 + static_cast<int>((static_cast<int64_t>(c->T) * c->top_k + 31) / 32)
                      : 0;
    MOE_TRY(moe::dispatch_positions(topk_idx, blk, slot_pos, perm_src, c->T, c->top_k,
                                    c->n_experts, moe::kRankBlock, s,
                                    copy_counters ? at<int32_t>(ws, L.copy_ready) : nullptr,
                                    n_zero));
    return MOE_OK;
  }
  MOE_TRY(moe::dispatch_scatter(c->dtype == MOE_BF16, x, topk_idx, blk, slot_pos, perm_src,
                                x_perm, c->T, c->d_model, c->top_k, c->n_experts,
                                moe::kRankBlock, s));
  return MOE_OK;
}

// Optional CUDA events recorded between the phases of moe_forward_profiled.
struct Marks {
  void* const* ev;
  cudaStream_t s;
  bool rec(int i) const {
    return ev == nullptr || cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), s) == cudaSuccess;
  }
};

// x_perm == nullptr (bf16 only): the gate/up GEMM gathers its rows from x
// through gather_rows (perm_src) instead of reading a permuted copy.
// fold (bf16 only): the down GEMM also forms the combined output.
// copy (bf16 only, with x_perm): the gate/up GEMM fills x_perm itself.
moe_status run_experts(const moe_config* c, const void* x_perm, const int32_t* offsets,
                       const moe_expert_weights* w, const void* x, void* y_perm, void* y_shared,
                       void* ws, cudaStream_t s, const Marks& mk,
                       const int32_t* gather_rows = nullptr,
                       const moe::GemmFold* fold = nullptr,
                       const moe::GemmCopy* copy = nullptr) {
  const Layout L = layout(*c);
  uint32_t* status = at<uint32_t>(ws, L.status);
  const int64_t R = static_cast<int64_t>(c->T) * c->top_k;
  const int E = c->n_experts, F = c->d_ff, d = c->d_model;
  void* h = at<void>(ws, L.h);
  if (c->dtype == MOE_BF16) {
    // the shared expert runs as one more group of the routed launches
    void* hs = at<void>(ws, L.h_sh);
    const int Fs = c->d_ff_shared;
    const moe::GemmExtraGroup sh_up{x, c->T, w->ws1, w->ws3, Fs, d, hs};
    const moe::GemmExtraGroup sh_down{hs, c->T, w->ws2, nullptr, d, Fs, y_shared};
    if (x_perm == nullptr) {
      MOE_TRY(moe::grouped_swiglu_gateup_gather_bf16(x, c->T, gather_rows, R, offsets, E, w->w1,
                                                     w->w3, F, d, h, status, s,
                                                     c->n_shared ? &sh_up : nullptr));
    } else {
      MOE_TRY(moe::grouped_swiglu_gateup_bf16(x_perm, R, offsets, E, 0, w->w1, w->w3, F, d, h,
                                              status, s, c->n_shared ? &sh_up : nullptr,
                                              copy));
    }
    if (!mk.rec(3)) return MOE_ERR_CUDA;
    MOE_TRY(moe::grouped_down_bf16(h, R, offsets, E, 0, w->w2, d, F, y_perm, status, s,
                                   c->n_shared ? &sh_down : nullptr, fold));
    if (!mk.rec(4)) return MOE_ERR_CUDA;
  } else {
    float* hf = static_cast<float*>(h);
    MOE_TRY(moe::grouped_swiglu_gateup_f32(static_cast<const float*>(x_perm), R, offsets, E, 0,
                                           static_cast<const float*>(w->w1),
                                           static_cast<const float*>(w->w3), F, d, hf, s));
    if (!mk.rec(3)) return MOE_ERR_CUDA;
    MOE_TRY(moe::grouped_down_f32(hf, R, offsets, E, 0, static_cast<const float*>(w->w2), d, F,
                                  static_cast<float*>(y_perm), s));
    if (!mk.rec(4)) return MOE_ERR_CUDA;
    if (c->n_shared) {
      float* hs = at<float>(ws, L.h_sh);
      const int Fs = c->d_ff_shared;
      MOE_TRY(moe::grouped_swiglu_gateup_f32(static_cast<const float*>(x), c->T, nullptr, 1,
                                             c->T, static_cast<const float*>(w->ws1),
                                             static_cast<const float*>(w->ws3), Fs, d, hs, s));
      MOE_TRY(moe::grouped_down_f32(hs, c->T, nullptr, 1, c->T,
                                    static_cast<const float*>(w->ws2), d, Fs,
                                    static_cast<float*>(y_shared), s));
    }
  }
  if (!mk.rec(5)) return MOE_ERR_CUDA;
  return MOE_OK;
}

moe_status check_weights(const moe_config* c, const moe_expert_weights* w) {
  if (w == nullptr || !w->w1 || !w->w3 || !w->w2) return MOE_ERR_INVALID;
  if (!aligned16(w->w1) || !aligned16(w->w3) || !aligned16(w->w2)) return MOE_ERR_INVALID;
  if (c->n_shared) {
    if (!w->ws1 || !w->ws3 || !w->ws2) return MOE_ERR_INVALID;
    if (!aligned16(w->ws1) || !aligned16(w->ws3) || !aligned16(w->ws2)) return MOE_ERR_INVALID;
  }
  return MOE_OK;
}

moe_status forward_impl(const moe_config* cfg, const void* x, const void* w_router,
                        const float* sel_bias, const float* logit_offset,
                        const moe_expert_weights* w, void* out, int32_t* topk_idx,
                        float* topk_w, int32_t* counts, void* ws, size_t ws_bytes, void* stream,
                        void* const* events, const moe_forward_opts* opts = nullptr) {
  moe_status st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  if (opts != nullptr &&
      ((opts->gather_rows != 0 && opts->gather_rows != 1) ||
       (opts->fold_combine != 0 && opts->fold_combine != 1) ||
       (opts->scatter_in_gemm != 0 && opts->scatter_in_gemm != 1) || opts->reserved[0] != 0 ||
       (opts->gather_rows == 1 && opts->scatter_in_gemm == 1)))
    return MOE_ERR_INVALID;
  const bool gather = opts != nullptr && opts->gather_rows == 1;
  const bool fold = opts != nullptr && opts->fold_combine == 1;
  const bool scat = opts != nullptr && opts->scatter_in_gemm == 1;
  if ((gather || fold || scat) && cfg->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (!counts) return MOE_ERR_INVALID;
  if (cfg->T == 0) {
    MOE_TRY(cudaMemsetAsync(counts, 0, sizeof(int32_t) * cfg->n_experts, S(stream)));
    return MOE_OK;
  }
  if (!x || !w_router || !out || !topk_idx || !topk_w) return MOE_ERR_INVALID;
  if ((st = check_weights(cfg, w)) != MOE_OK) return st;
  if (!aligned16(x) || !aligned16(w_router) || !aligned16(out) || !aligned4(topk_idx) ||
      !aligned4(topk_w) || !aligned4(counts) || (sel_bias && !aligned4(sel_bias)) ||
      (logit_offset && !aligned4(logit_offset)))
    return MOE_ERR_INVALID;
  if (events)
    for (int i = 0; i <= MOE_FORWARD_PHASES; ++i)
      if (!events[i]) return MOE_ERR_INVALID;
  if ((st = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return st;
  const Layout L = layout(*cfg);
  cudaStream_t s = S(stream);
  const Marks mk{events, s};
  if ((st = clear_status(ws, s)) != MOE_OK) return st;
  if (!mk.rec(0)) return MOE_ERR_CUDA;
  if ((st = run_router(cfg, x, w_router, sel_bias, logit_offset, topk_idx, topk_w, ws, s)) !=
      MOE_OK)
    return st;
  if (!mk.rec(1)) return MOE_ERR_CUDA;
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* slot_pos = at<int32_t>(ws, L.slot_pos);
  void* x_perm = at<void>(ws, L.x_perm);
  void* y_perm = at<void>(ws, L.y_perm);
  void* y_sh = cfg->n_shared ? at<void>(ws, L.y_sh) : nullptr;
  // Default: dispatch writes the permuted copy x_perm and the gate/up GEMM
  // reads it with TMA tiles.  opts->gather_rows (bf16 only) skips the copy
  // and lets the gate/up GEMM gather its rows from x by perm_src; it moves
  // less memory but measured slower on B200 (each of an m-tile's n-tile CTAs
  // gathers the same rows again).
  int32_t* perm_src = at<int32_t>(ws, L.perm_src);
  if (gather) MOE_TRY(cudaMemsetAsync(at<uint32_t>(ws, L.status) + 2, 0xff, sizeof(uint32_t), s));
  // fold_combine: the down GEMM's epilogue forms out (dispatch sets its
  // per-token counts); no combine launch
  const int fold_nt =
      fold ? (cfg->d_model + moe::down_tile_cols(cfg->d_model, cfg->d_ff) - 1) /
                 moe::down_tile_cols(cfg->d_model, cfg->d_ff)
           : 0;
  // scatter_in_gemm: dispatch writes the rows' positions only, and the
  // gate/up GEMM copies x's rows into x_perm while it runs
  if ((st = run_permute(cfg, topk_idx, x, counts, offsets, slot_pos, perm_src,
                        (gather || scat) ? nullptr : x_perm, ws, s, fold_nt, scat)) != MOE_OK)
    return st;
  if (!mk.rec(2)) return MOE_ERR_CUDA;
  const moe::GemmFold gf{at<int32_t>(ws, L.fold), fold_nt, cfg->T, cfg->top_k, perm_src,
                         slot_pos, topk_w, out};
  const moe::GemmCopy gc{x, cfg->T, perm_src, at<int32_t>(ws, L.copy_ready)};
  if ((st = run_experts(cfg, gather ? nullptr : x_perm, offsets, w, x, y_perm, y_sh, ws, s, mk,
                        perm_src, fold ? &gf : nullptr, scat ? &gc : nullptr)) != MOE_OK)
    return st;
  if (!fold)
    MOE_TRY(moe::combine(cfg->dtype == MOE_BF16, y_perm, slot_pos, topk_w, y_sh, out, cfg->T,
                         cfg->d_model, cfg->top_k, s));
  if (!mk.rec(MOE_FORWARD_PHASES)) return MOE_ERR_CUDA;
  return MOE_OK;
}

// Workspace of moe_backward (separate from the forward's, which it reads).
struct BLayout {
  size_t status, dw, logits, dlogits, adx, adw, wr3, pdw, goff, dxr, dy, dh, dgu, dxp, dh_sh,
      dgu_sh, dxs, total;
};

BLayout blayout(const moe_config& c) {
  const size_t T = static_cast<size_t>(c.T), d = c.d_model, E = c.n_experts, F = c.d_ff,
               k = c.top_k, R = T * k;
  const size_t Fs = c.n_shared ? static_cast<size_t>(c.d_ff_shared) : 0;
  BLayout B{};
  size_t o = 0;
  B.status = o;  o += up(2 * sizeof(uint32_t));
  B.dw = o;      o += up(R * 4);
  B.logits = o;  o += up(T * E * 4);
  B.dlogits = o; o += up(T * E * 4);
  const moe::RouterGradShape rg = moe::router_grad_shape(c.T, c.n_experts);
  const size_t C3 = 3 * static_cast<size_t>(rg.Ep), Gs = rg.G, Ks = rg.Ks;
  B.adx = o;     o += up(T * C3 * 2);
  B.adw = o;     o += up(Gs * C3 * Ks * 2);
  B.wr3 = o;     o += up(C3 * d * 2);
  B.pdw = o;     o += up(Gs * C3 * d * 4);
  B.goff = o;    o += up((Gs + 1) * 4);
  B.dxr = o;     o += up(T * d * 4);
  B.dy = o;      o += up(R * d * 2);
  B.dh = o;      o += up(R * F * 2);
  B.dgu = o;     o += up(R * 2 * F * 2);
  B.dxp = o;     o += up(R * d * 2);
  B.dh_sh = o;   o += up(T * Fs * 2);
  B.dgu_sh = o;  o += up(T * 2 * Fs * 2);
  B.dxs = o;     o += up(Fs ? T * d * 2 : 0);
  B.total = o;
  return B;
}

// The layer's backward (bf16 layers).  fws holds the state of the forward:
// offsets, slot_pos, perm_src, x_perm (unless that forward gathered its rows:
// status word 2), h, y_perm (and h_sh).
moe_status backward_impl(const moe_config* c, const void* x, const void* w_router,
                         const float* logit_offset, const moe_expert_weights* w,
                         const int32_t* topk_idx, const float* topk_w, const void* dout,
                         void* dx, float* dw_router, const moe_expert_grads* g, void* fws,
                         void* bws, cudaStream_t s) {
  const Layout L = layout(*c);
  const BLayout B = blayout(*c);
  const int T = c->T, d = c->d_model, E = c->n_experts, F = c->d_ff, k = c->top_k;
  const int64_t R = static_cast<int64_t>(T) * k;
  uint32_t* status = at<uint32_t>(bws, B.status);
  const int32_t* offsets = at<int32_t>(fws, L.offsets);
  const int32_t* slot_pos = at<int32_t>(fws, L.slot_pos);
  const int32_t* perm_src = at<int32_t>(fws, L.perm_src);
  const void* h = at<void>(fws, L.h);
  const void* y_perm = at<void>(fws, L.y_perm);
  float* dw = at<float>(bws, B.dw);
  // combine: dw and the experts' output gradients
  MOE_TRY(moe::bwd_dy(dout, y_perm, slot_pos, topk_w, at<void>(bws, B.dy), dw, T, d, k, s));
  // dH = dY W2 ; G, U recomputed ; dG, dU ; dX = [dG | dU] [W1 ; W3].  The
  // weights of dH and dX are read MN-major in place (no transposed copies).
  MOE_TRY(moe::grouped_gemm_bmn_bf16(at<void>(bws, B.dy), R, offsets, E, 0, w->w2, nullptr, d,
                                     F, d, at<void>(bws, B.dh), status, s));
  // x's rows in expert order: the forward's x_perm, written here from x by
  // the permutation when that forward gathered its rows instead (status
  // word 2 set).  G and U are recomputed from it on the tensor cores, and the
  // SwiGLU backward runs in that GEMM's epilogue: [dG | dU] from G, U, dH.
  void* x_perm = at<void>(fws, L.x_perm);
  MOE_TRY(moe::fill_xperm(x, perm_src, at<uint32_t>(fws, L.status) + 2, x_perm, R, T, d, s));
  MOE_TRY(moe::grouped_swiglu_bwd_bf16(x_perm, R, offsets, E, 0, w->w1, w->w3, F, d,
                                       at<void>(bws, B.dh), at<void>(bws, B.dgu), status, s));
  MOE_TRY(moe::grouped_gemm_bmn_bf16(at<void>(bws, B.dgu), R, offsets, E, 0, w->w1, w->w3, F, d,
                                     2 * F, at<void>(bws, B.dxp), status, s));
  // weight gradients over each expert's rows, the row-major activations
  // read MN-major: dW2 = dY^T h, dW1 = dG^T x_perm, dW3 = dU^T x_perm
  MOE_TRY(moe::grouped_wgrad_bf16(at<void>(bws, B.dy), d, 0, h, F, 0, R, offsets, E, d, F,
                                  g->dw2, status, s));
  MOE_TRY(moe::grouped_wgrad_bf16(at<void>(bws, B.dgu), 2 * F, 0, x_perm, d, 0, R, offsets, E, F,
                                  d, g->dw1, status, s));
  MOE_TRY(moe::grouped_wgrad_bf16(at<void>(bws, B.dgu), 2 * F, F, x_perm, d, 0, R, offsets, E, F,
                                  d, g->dw3, status, s));
  // shared expert (weight 1, all tokens)
  const void* dxs = nullptr;
  if (c->n_shared) {
    const int Fs = c->d_ff_shared;
    MOE_TRY(moe::grouped_gemm_bmn_bf16(dout, T, nullptr, 1, T, w->ws2, nullptr, d, Fs, d,
                                       at<void>(bws, B.dh_sh), status, s));
    MOE_TRY(moe::grouped_swiglu_bwd_bf16(x, T, nullptr, 1, T, w->ws1, w->ws3, Fs, d,
                                         at<void>(bws, B.dh_sh), at<void>(bws, B.dgu_sh), status,
                                         s));
    MOE_TRY(moe::grouped_gemm_bmn_bf16(at<void>(bws, B.dgu_sh), T, nullptr, 1, T, w->ws1,
                                       w->ws3, Fs, d, 2 * Fs, at<void>(bws, B.dxs), status, s));
    dxs = at<void>(bws, B.dxs);
    MOE_TRY(moe::grouped_wgrad_bf16(dout, d, 0, at<void>(fws, L.h_sh), Fs, 0, T, nullptr, 1, d,
                                    Fs, g->dws2, status, s));
    MOE_TRY(moe::grouped_wgrad_bf16(at<void>(bws, B.dgu_sh), 2 * Fs, 0, x, d, 0, T, nullptr, 1,
                                    Fs, d, g->dws1, status, s));
    MOE_TRY(moe::grouped_wgrad_bf16(at<void>(bws, B.dgu_sh), 2 * Fs, Fs, x, d, 0, T, nullptr, 1,
                                    Fs, d, g->dws3, status, s));
  }
  // router (fp32): recomputed logits, dlogits, then on the tensor cores
  // with dlogits as three exact bf16 terms: dx_router = dlogits Wr (K = 3 Ep,
  // Wr repeated per term) and dW_router = dlogits^T x (G token slices as
  // GEMM groups, fp32 partials summed in a fixed order)
  float* logits = at<float>(bws, B.logits);
  float* dlogits = at<float>(bws, B.dlogits);
  MOE_TRY(moe::router_logits_tc(x, T, w_router, E, d, logits, status, s));
  MOE_TRY(moe::router_dlogits(logits, logit_offset, topk_idx, topk_w, dw, T, E, k, c->gate,
                              c->norm_topk_prob, dlogits, s));
  const moe::RouterGradShape rg = moe::router_grad_shape(T, E);
  const int C3 = 3 * rg.Ep;
  uint8_t* wr3 = at<uint8_t>(bws, B.wr3);
  const size_t wr_bytes = static_cast<size_t>(E) * d * 2;
  for (int j = 0; j < 3; ++j) {
    uint8_t* dst = wr3 + static_cast<size_t>(j) * rg.Ep * d * 2;
    MOE_TRY(cudaMemcpyAsync(dst, w_router, wr_bytes, cudaMemcpyDeviceToDevice, s));
    if (rg.Ep > E)
      MOE_TRY(cudaMemsetAsync(dst + wr_bytes, 0, static_cast<size_t>(rg.Ep - E) * d * 2, s));
  }
  MOE_TRY(moe::router_grad_split(dlogits, T, E, rg, at<void>(bws, B.adx), at<void>(bws, B.adw),
                                 at<int32_t>(bws, B.goff), s));
  MOE_TRY(moe::grouped_gemm_bmn_f32out(at<void>(bws, B.adx), T, nullptr, 1, T, wr3, C3, C3, d,
                                       at<float>(bws, B.dxr), status, s));
  MOE_TRY(moe::grouped_gemm_bmn_f32out(at<void>(bws, B.adw), static_cast<int64_t>(rg.G) * C3,
                                       at<int32_t>(bws, B.goff), rg.G, 0, x, rg.Ks, T, d,
                                       at<float>(bws, B.pdw), status, s));
  MOE_TRY(moe::router_grad_reduce(at<float>(bws, B.pdw), rg, E, d, dw_router, s));
  MOE_TRY(moe::dx_gather(at<void>(bws, B.dxp), slot_pos, at<float>(bws, B.dxr), dxs, dx, T, d, k,
                         s));
  return MOE_OK;
}

}  // namespace

extern "C" {

size_t moe_workspace_size(const moe_config* cfg) {
  if (check_cfg(cfg) != MOE_OK) return 0;
  return layout(*cfg).total;
}

moe_status moe_check_config(const moe_config* cfg) { return check_cfg(cfg); }

moe_status moe_router_topk(const moe_config* cfg, const void* x, const void* w_router,
                           const float* sel_bias, const float* logit_offset, int32_t* topk_idx,
                           float* topk_w, void* ws, size_t ws_bytes, void* stream) {
  moe_status st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) return MOE_OK;
  if (!x || !w_router || !topk_idx || !topk_w) return MOE_ERR_INVALID;
  if (!aligned16(x) || !aligned16(w_router) || !aligned4(topk_idx) || !aligned4(topk_w) ||
      (sel_bias && !aligned4(sel_bias)) || (logit_offset && !aligned4(logit_offset)))
    return MOE_ERR_INVALID;
  if ((st = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return st;
  if ((st = clear_status(ws, S(stream))) != MOE_OK) return st;
  return run_router(cfg, x, w_router, sel_bias, logit_offset, topk_idx, topk_w, ws, S(stream));
}

moe_status moe_router_topk_opts(const moe_config* cfg, const void* x, const void* w_router,
                                const float* sel_bias, const float* logit_offset,
                                const moe_router_opts* opts, int32_t* topk_idx, float* topk_w,
                                void* ws, size_t ws_bytes, void* stream) {
  if (opts == nullptr || (opts->bias_space != 0 && opts->bias_space != 1) ||
      (opts->sel_noise && !aligned4(opts->sel_noise)))
    return MOE_ERR_INVALID;
  moe_status st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) return MOE_OK;
  if (!x || !w_router || !topk_idx || !topk_w) return MOE_ERR_INVALID;
  if (!aligned16(x) || !aligned16(w_router) || !aligned4(topk_idx) || !aligned4(topk_w) ||
      (sel_bias && !aligned4(sel_bias)) || (logit_offset && !aligned4(logit_offset)))
    return MOE_ERR_INVALID;
  if ((st = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return st;
  if ((st = clear_status(ws, S(stream))) != MOE_OK) return st;
  moe::KeyOpts ko;
  ko.space = opts->bias_space;
  ko.noise = opts->sel_noise;
  return run_router(cfg, x, w_router, sel_bias, logit_offset, topk_idx, topk_w, ws, S(stream),
                    ko);
}

moe_status moe_router_logits(const moe_config* cfg, const void* x, const void* w_router,
                             const float* logit_offset, float* logits, void* ws,
                             size_t ws_bytes, void* stream) {
  moe_status st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  if (cfg->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (cfg->T == 0) return MOE_OK;
  if (!x || !w_router || !logits || !aligned16(x) || !aligned16(w_router) || !aligned4(logits) ||
      (logit_offset && !aligned4(logit_offset)))
    return MOE_ERR_INVALID;
  if ((st = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return st;
  if ((st = clear_status(ws, S(stream))) != MOE_OK) return st;
  MOE_TRY(moe::router_logits_tc(x, cfg->T, w_router, cfg->n_experts, cfg->d_model, logits,
                                at<uint32_t>(ws, 0), S(stream)));
  if (logit_offset)
    MOE_TRY(moe::add_row_offset(logits, logit_offset, cfg->T, cfg->n_experts, S(stream)));
  return MOE_OK;
}

moe_status moe_router_stats(const moe_config* cfg, const void* x, const void* w_router,
                            const float* logit_offset, const int32_t* topk_idx, float* stats,
                            void* ws, size_t ws_bytes, void* stream) {
  moe_status st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  if (!stats || !aligned4(stats)) return MOE_ERR_INVALID;
  if (cfg->T == 0) {
    MOE_TRY(cudaMemsetAsync(stats, 0, 8 * sizeof(float), S(stream)));
    return MOE_OK;
  }
  if (!x || !w_router || !topk_idx || !aligned16(x) || !aligned16(w_router) ||
      !aligned4(topk_idx) || (logit_offset && !aligned4(logit_offset)))
    return MOE_ERR_INVALID;
  if ((st = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return st;
  const Layout L = layout(*cfg);
  cudaStream_t s = S(stream);
  if ((st = clear_status(ws, s)) != MOE_OK) return st;
  void* logits = at<void>(ws, L.logits);
  const bool bf16 = cfg->dtype == MOE_BF16;
  if (bf16) {
    MOE_TRY(moe::router_logits_tc(x, cfg->T, w_router, cfg->n_experts, cfg->d_model,
                                  static_cast<float*>(logits), at<uint32_t>(ws, 0), s));
    if (logit_offset)
      MOE_TRY(moe::add_row_offset(static_cast<float*>(logits), logit_offset, cfg->T,
                                  cfg->n_experts, s));
  } else {
    MOE_TRY(moe::router_logits(false, x, w_router, logit_offset, cfg->T, cfg->d_model,
                               cfg->n_experts, static_cast<double*>(logits), s));
  }
  MOE_TRY(moe::router_stats(!bf16, logits, cfg->T, cfg->n_experts, cfg->gate, topk_idx,
                            cfg->top_k, at<double>(ws, L.stats), stats, s));
  return MOE_OK;
}

moe_status moe_permute(const moe_config* cfg, const int32_t* topk_idx, const void* x,
                       int32_t* counts, int32_t* offsets, int32_t* slot_pos, int32_t* perm_src,
                       void* x_perm, void* ws, size_t ws_bytes, void* stream) {
  moe_status st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  if (!counts || !offsets) return MOE_ERR_INVALID;
  if (cfg->T == 0) {
    MOE_TRY(cudaMemsetAsync(counts, 0, sizeof(int32_t) * cfg->n_experts, S(stream)));
    MOE_TRY(cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (cfg->n_experts + 1), S(stream)));
    return MOE_OK;
  }
  if (!topk_idx || !x || !slot_pos || !perm_src || !x_perm) return MOE_ERR_INVALID;
  if (!aligned16(x) || !aligned16(x_perm) || !aligned4(topk_idx) || !aligned4(counts) ||
      !aligned4(offsets) || !aligned4(slot_pos) || !aligned4(perm_src))
    return MOE_ERR_INVALID;
  if ((st = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return st;
  if ((st = clear_status(ws, S(stream))) != MOE_OK) return st;
  return run_permute(cfg, topk_idx, x, counts, offsets, slot_pos, perm_src, x_perm, ws,
                     S(stream));
}

moe_status moe_grouped_swiglu(const moe_config* cfg, const void* x_perm, const int32_t* offsets,
                              const moe_expert_weights* w, const void* x, void* y_perm,
                              void* y_shared, void* ws, size_t ws_bytes, void* stream) {
  moe_status st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) return MOE_OK;
  if (!x_perm || !offsets || !y_perm) return MOE_ERR_INVALID;
  if ((st = check_weights(cfg, w)) != MOE_OK) return st;
  if (cfg->n_shared && (!x || !y_shared)) return MOE_ERR_INVALID;
  if (!cfg->n_shared && y_shared) return MOE_ERR_INVALID;
  if (!aligned16(x_perm) || !aligned16(y_perm) || !aligned4(offsets) ||
      (x && !aligned16(x)) || (y_shared && !aligned16(y_shared)))
    return MOE_ERR_INVALID;
  if ((st = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return st;
  if ((st = clear_status(ws, S(stream))) != MOE_OK) return st;
  return run_experts(cfg, x_perm, offsets, w, x, y_perm, y_shared, ws, S(stream),
                     Marks{nullptr, S(stream)});
}

moe_status moe_combine(const moe_config* cfg, const void* y_perm, const int32_t* slot_pos,
                       const float* topk_w, const void* y_shared, void* out, void* stream) {
  moe_status st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) return MOE_OK;
  if (!y_perm || !slot_pos || !topk_w || !out) return MOE_ERR_INVALID;
  if (cfg->n_shared && !y_shared) return MOE_ERR_INVALID;
  if (!cfg->n_shared && y_shared) return MOE_ERR_INVALID;
  if (!aligned16(y_perm) || !aligned16(out) || !aligned4(slot_pos) || !aligned4(topk_w) ||
      (y_shared && !aligned16(y_shared)))
    return MOE_ERR_INVALID;
  MOE_TRY(moe::combine(cfg->dtype == MOE_BF16, y_perm, slot_pos, topk_w, y_shared, out, cfg->T,
                       cfg->d_model, cfg->top_k, S(stream)));
  return MOE_OK;
}

moe_status moe_bias_update(const moe_config* cfg, const int32_t* counts, float* sel_bias,
                           double rate, double starved_frac, double starved_add, double clamp,
                           void* stream) {
  moe_status st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  if (!counts || !sel_bias || !aligned4(counts) || !aligned4(sel_bias)) return MOE_ERR_INVALID;
  if (!(clamp >= 0.0)) return MOE_ERR_INVALID;
  const double inv_e = 1.0 / static_cast<double>(cfg->n_experts);
  MOE_TRY(moe::bias_update(counts, sel_bias, cfg->n_experts, static_cast<float>(inv_e),
                           static_cast<float>(starved_frac * inv_e),
                           static_cast<float>(starved_add), static_cast<float>(rate),
                           static_cast<float>(clamp), S(stream)));
  return MOE_OK;
}

moe_status moe_bias_update_sign(const moe_config* cfg, const int32_t* counts, float* sel_bias,
                                double rate, void* stream) {
  moe_status st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  if (!counts || !sel_bias || !aligned4(counts) || !aligned4(sel_bias)) return MOE_ERR_INVALID;
  MOE_TRY(moe::bias_update_sign(counts, sel_bias, cfg->n_experts, static_cast<float>(rate),
                                S(stream)));
  return MOE_OK;
}

moe_status moe_forward(const moe_config* cfg, const void* x, const void* w_router,
                       const float* sel_bias, const float* logit_offset,
                       const moe_expert_weights* w, void* out, int32_t* topk_idx, float* topk_w,
                       int32_t* counts, void* ws, size_t ws_bytes, void* stream) {
  return forward_impl(cfg, x, w_router, sel_bias, logit_offset, w, out, topk_idx, topk_w, counts,
                      ws, ws_bytes, stream, nullptr);
}

moe_status moe_forward_profiled(const moe_config* cfg, const void* x, const void* w_router,
                                const float* sel_bias, const float* logit_offset,
                                const moe_expert_weights* w, void* out, int32_t* topk_idx,
                                float* topk_w, int32_t* counts, void* ws, size_t ws_bytes,
                                void* stream, void* const* events) {
  if (events == nullptr) return MOE_ERR_INVALID;
  return forward_impl(cfg, x, w_router, sel_bias, logit_offset, w, out, topk_idx, topk_w, counts,
                      ws, ws_bytes, stream, events);
}

moe_status moe_forward_ex(const moe_config* cfg, const void* x, const void* w_router,
                          const float* sel_bias, const float* logit_offset,
                          const moe_expert_weights* w, void* out, int32_t* topk_idx,
                          float* topk_w, int32_t* counts, const moe_forward_opts* opts, void* ws,
                          size_t ws_bytes, void* stream) {
  if (opts == nullptr) return MOE_ERR_INVALID;
  return forward_impl(cfg, x, w_router, sel_bias, logit_offset, w, out, topk_idx, topk_w, counts,
                      ws, ws_bytes, stream, nullptr, opts);
}

moe_status moe_forward_dispatch_view(const moe_config* cfg, const void* ws, size_t ws_bytes,
                                     const int32_t** offsets, const int32_t** slot_pos,
                                     const int32_t** perm_src) {
  moe_status st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  if (!offsets || !slot_pos || !perm_src) return MOE_ERR_INVALID;
  if ((st = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return st;
  const Layout L = layout(*cfg);
  void* base = const_cast<void*>(ws);
  *offsets = at<int32_t>(base, L.offsets);
  *slot_pos = at<int32_t>(base, L.slot_pos);
  *perm_src = at<int32_t>(base, L.perm_src);
  return MOE_OK;
}

moe_status moe_device_status(void* ws, size_t ws_bytes, void* stream, uint32_t* flags) {
  if (ws == nullptr || ws_bytes < sizeof(uint32_t)) return MOE_ERR_INVALID;
  uint32_t v = 0;
  MOE_TRY(cudaStreamSynchronize(S(stream)));
  MOE_TRY(cudaMemcpy(&v, ws, sizeof(v), cudaMemcpyDeviceToHost));
  MOE_TRY(cudaMemset(ws, 0, sizeof(v)));
  if (flags) *flags = v;
  if (v & moe::kDevTimeout) return MOE_ERR_TIMEOUT;
  if (v & moe::kDevBadIndex) return MOE_ERR_DATA;
  return MOE_OK;
}

moe_status moe_router_refined_tokens(void* ws, size_t ws_bytes, void* stream, int32_t* count) {
  if (ws == nullptr || ws_bytes < 2 * sizeof(int32_t) || count == nullptr) return MOE_ERR_INVALID;
  MOE_TRY(cudaStreamSynchronize(S(stream)));
  MOE_TRY(cudaMemcpy(count, static_cast<int32_t*>(ws) + 1, sizeof(int32_t),
                     cudaMemcpyDeviceToHost));
  return MOE_OK;
}

size_t moe_backward_workspace_size(const moe_config* cfg) {
  if (check_cfg(cfg) != MOE_OK || cfg->dtype != MOE_BF16) return 0;
  return blayout(*cfg).total;
}

moe_status moe_backward(const moe_config* cfg, const void* x, const void* w_router,
                        const float* logit_offset, const moe_expert_weights* w,
                        const int32_t* topk_idx, const float* topk_w, const void* dout, void* dx,
                        float* dw_router, const moe_expert_grads* g, void* fws, size_t fws_bytes,
                        void* bws, size_t bws_bytes, void* stream) {
  moe_status st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  if (cfg->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (cfg->T == 0) return MOE_OK;
  if (!x || !w_router || !topk_idx || !topk_w || !dout || !dx || !dw_router || !g || !g->dw1 ||
      !g->dw3 || !g->dw2 || (cfg->n_shared && (!g->dws1 || !g->dws3 || !g->dws2)))
    return MOE_ERR_INVALID;
  if ((st = check_weights(cfg, w)) != MOE_OK) return st;
  if (!aligned16(x) || !aligned16(w_router) || !aligned16(dout) || !aligned16(dx) ||
      !aligned16(dw_router) || !aligned4(topk_idx) || !aligned4(topk_w) || !aligned16(g->dw1) ||
      !aligned16(g->dw3) || !aligned16(g->dw2) || (logit_offset && !aligned4(logit_offset)) ||
      (cfg->n_shared && (!aligned16(g->dws1) || !aligned16(g->dws3) || !aligned16(g->dws2))))
    return MOE_ERR_INVALID;
  if ((st = check_ws(cfg, fws, fws_bytes)) != MOE_OK) return st;
  if (bws == nullptr || (reinterpret_cast<uintptr_t>(bws) & (kAlign - 1))) return MOE_ERR_INVALID;
  if (bws_bytes < blayout(*cfg).total) return MOE_ERR_WORKSPACE;
  cudaStream_t s = S(stream);
  if ((st = clear_status(bws, s)) != MOE_OK) return st;
  return backward_impl(cfg, x, w_router, logit_offset, w, topk_idx, topk_w, dout, dx, dw_router,
                       g, fws, bws, s);
}

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "configuration outside the supported limits";
    case MOE_ERR_WORKSPACE: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA runtime error";
    case MOE_ERR_TIMEOUT: return "a bounded device wait gave up";
    case MOE_ERR_DATA: return "expert index outside [0, E) or repeated within a token";
  }
  return "unknown status";
}

}  // extern "C"
