"""CPU oracle for the MoE FFN layer: forward, backward, router statistics and
the selection-bias updates.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or run
this module: only the tests, the smoke check and the benchmark's CPU-baseline
leg use it.  It shares no code with the CUDA library (no kernels, headers,
helpers or constants); the only thing both sides read is the seeded input
generator, which holds none of the layer's arithmetic.

Everything is the plain definition of the layer, evaluated in float64 on the
(bf16- or fp32-valued) inputs, one step per stated operation, with numpy's
matmul and sort as the only library primitives.  The bias update is the one
step computed in float32, because the pages fix its arithmetic to an fp32
buffer and the result is compared bit for bit.

Sources (page title, section):

* "moe-200m-qwen3-100b" README, section "SigmoidRouter (the patched, DDP-safe
  router)": fp32 router linear, sigmoid scores, selection logits = logits +
  bias, top-k of the selection logits, combine weights gathered from the
  *unbiased* scores and divided by (their sum + 1e-9); ``step_bias_update``:
  magnitude controller with the starved-expert boost and the +-10 clamp.
* same README, "Architecture diagram": router -> top-k routing -> routed
  SwiGLU experts + one always-on shared SwiGLU expert -> weighted sum.
* same README, "Per-layer numerics": the router runs in fp32 with autocast off.
* "SpecForge PR #930 (qwen3 MoE preset)", "What this adds": softmax over all
  experts, top-k combine weights renormalised (norm_topk_prob), no scaling, no
  shared expert, plain SwiGLU; experts stacked as [E, out, in].
* "SpecForge PR #931 (MoE FFN for DFlash-family drafters)", "What works": the
  per-expert keys w1, w2, w3 and grouped-GEMM dispatch checked against a
  sorted loop over experts.

Readings of points the pages leave open (each one is listed with its reason in
the design notes of the repository):

* the selection bias is added to the logits for both gates;
* top-k order is descending key, equal keys go to the lower expert index;
* the renormalisation epsilon is 1e-9 for both gates;
* SwiGLU expert:  w2 @ (silu(w1 @ x) * (w3 @ x)),  silu(z) = z / (1 + e^-z);
  w1 = gate [F, d], w3 = up [F, d], w2 = down [d, F];
* the shared expert's output is added with weight 1, routed weights are not
  scaled;
* no capacity factor: every (token, choice) pair is computed;
* the expert-contiguous order is the stable sort of pairs by (expert, token).
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Sequence

import numpy as np

GATE_SOFTMAX = 0
GATE_SIGMOID = 1


@dataclasses.dataclass
class Routing:
    logits: np.ndarray     # [T, E] f64, router logits (+ per-expert offset if any)
    scores: np.ndarray     # [T, E] f64, gate scores (sigmoid or softmax)
    keys: np.ndarray       # [T, E] f64, selection keys = logits + bias
    topk_idx: np.ndarray   # [T, k] int64, descending key, ties to lower index
    topk_w: np.ndarray     # [T, k] f64, combine weights
    edge_gap: np.ndarray   # [T] f64, key_(k) - key_(k+1) (inf when k == E)
    min_gap: np.ndarray    # [T] f64, smallest adjacent gap among the top k+1 keys


def _as64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


def sigmoid(z: np.ndarray) -> np.ndarray:
    """1 / (1 + e^-z), evaluated without overflow warnings."""
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-z))


def silu(z: np.ndarray) -> np.ndarray:
    """SiLU / swish: z * sigmoid(z) = z / (1 + e^-z)."""
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def softmax_rows(z: np.ndarray) -> np.ndarray:
    """Softmax over the last axis, with the row maximum subtracted first."""
    m = z.max(axis=-1, keepdims=True)
    e = np.exp(z - m)
    return e / e.sum(axis=-1, keepdims=True)


def router(x, w_router, top_k: int, gate: int, norm_topk_prob: bool,
           sel_bias=None, logit_offset=None, bias_space: int = 0, sel_noise=None) -> Routing:
    """Router forward: logits, gate scores, biased selection, top-k, weights.

    Follows ``SigmoidRouter.forward`` ("moe-200m-qwen3-100b" README) for the
    sigmoid gate and the qwen3 preset (SpecForge PR #930, "What this adds") for
    the softmax gate.  ``logit_offset`` is a per-expert constant added to the
    logits before the gate (used only by the skewed-load workload).

    Selection-key variants: ``bias_space=1`` adds the bias to the gate scores
    instead of the logits (the score-space placement of the "noaux_tc" balance
    bias the page-3 model card names without code); ``sel_noise`` [T, E] is
    added to every key, the exploration noise of ``SigmoidRouter.forward``
    (``sel_logits += randn * noise_std``) with the draws and the scale
    supplied by the caller.  Both move the selection only.
    """
    x64, w64 = _as64(x), _as64(w_router)
    T, E = x64.shape[0], w64.shape[0]
    if not 1 <= top_k <= E:
        raise ValueError("top_k must be in [1, E]")
    # 1. logits = x . w_router^T  (fp32 router; evaluated here in fp64)
    logits = x64 @ w64.T
    if logit_offset is not None:
        logits = logits + _as64(logit_offset)[None, :]
    # 2. gate scores
    if gate == GATE_SIGMOID:
        scores = sigmoid(logits)
    elif gate == GATE_SOFTMAX:
        scores = softmax_rows(logits)
    else:
        raise ValueError("unknown gate")
    # 3. selection keys: the bias (and the noise) move the selection only
    if bias_space not in (0, 1):
        raise ValueError("bias_space must be 0 or 1")
    keys = logits if bias_space == 0 else scores
    if sel_bias is not None:
        keys = keys + _as64(sel_bias)[None, :]
    if sel_noise is not None:
        keys = keys + _as64(sel_noise)
    # 4. top-k: stable ascending sort of -key = descending key, ties -> lower e
    order = np.argsort(-keys, axis=1, kind="stable")
    idx = order[:, :top_k]
    # 5. combine weights from the unbiased scores, optionally renormalised
    w = np.take_along_axis(scores, idx, axis=1)
    if norm_topk_prob:
        w = w / (w.sum(axis=1, keepdims=True) + 1e-9)
    sorted_keys = np.take_along_axis(keys, order, axis=1)
    if top_k < E:
        edge = sorted_keys[:, top_k - 1] - sorted_keys[:, top_k]
        adj = sorted_keys[:, :top_k] - sorted_keys[:, 1:top_k + 1]
    else:
        edge = np.full(T, np.inf)
        adj = sorted_keys[:, :top_k - 1] - sorted_keys[:, 1:top_k]
    min_gap = adj.min(axis=1) if adj.shape[1] else np.full(T, np.inf)
    return Routing(logits, scores, keys, idx.astype(np.int64), w, edge, min_gap)


@dataclasses.dataclass
class Dispatch:
    counts: np.ndarray     # [E] int64: number of (t, j) pairs that chose e
    offsets: np.ndarray    # [E+1] int64: exclusive prefix sum of counts
    perm_src: np.ndarray   # [T*k] int64: token of the pair at each slot
    perm_expert: np.ndarray  # [T*k] int64: expert of the pair at each slot
    slot_pos: np.ndarray   # [T, k] int64: slot of pair (t, j)


def dispatch(topk_idx, n_experts: int) -> Dispatch:
    """Expert-contiguous order of the routed pairs.

    The rows that ``grouped_mm`` dispatch consumes (SpecForge PR #930 "Why FSDP
    is enough here"; PR #931 "What works": grouped GEMM vs a sorted loop): the
    pairs (t, j) sorted stably by (expert, token).
    """
    idx = np.asarray(topk_idx, dtype=np.int64)
    T, k = idx.shape
    flat = idx.reshape(-1)
    if flat.size and (flat.min() < 0 or flat.max() >= n_experts):
        raise ValueError("expert index out of range")
    counts = np.bincount(flat, minlength=n_experts).astype(np.int64)
    offsets = np.zeros(n_experts + 1, dtype=np.int64)
    np.cumsum(counts, out=offsets[1:])
    tok = np.repeat(np.arange(T, dtype=np.int64), k)
    order = np.lexsort((tok, flat))          # primary: expert, secondary: token
    slot_pos = np.empty(T * k, dtype=np.int64)
    slot_pos[order] = np.arange(T * k, dtype=np.int64)
    return Dispatch(counts, offsets, tok[order], flat[order], slot_pos.reshape(T, k))


def swiglu_expert(xr, w1, w3, w2) -> np.ndarray:
    """One SwiGLU expert on rows xr [n, d]:  (silu(xr w1^T) * (xr w3^T)) w2^T."""
    xr = _as64(xr)
    g = xr @ _as64(w1).T           # gate   [n, F]
    u = xr @ _as64(w3).T           # up     [n, F]
    return (silu(g) * u) @ _as64(w2).T   # down [n, d]


def moe_forward(inp: dict, top_k: int, gate: int, norm_topk_prob: bool,
                tokens: Optional[Sequence[int]] = None, routing: Optional[Routing] = None):
    """Layer output for the selected tokens (all tokens when ``tokens`` is None).

    out[t] = shared(x[t]) + sum_j w[t, j] * expert_{idx[t, j]}(x[t])
    ("moe-200m-qwen3-100b" README, "Architecture diagram": routed experts plus
    the always-on shared expert, then the weighted sum).  The routed part is a
    loop over experts on the rows sorted to each expert, the "sorted loop" that
    SpecForge PR #931 checks grouped GEMM dispatch against.
    Returns (out [n, d] f64, routing).
    """
    x = inp["x"]
    if routing is None:
        routing = router(x, inp["w_router"], top_k, gate, norm_topk_prob,
                         inp.get("sel_bias"), inp.get("logit_offset"))
    sel = np.arange(x.shape[0]) if tokens is None else np.asarray(tokens, dtype=np.int64)
    xs = _as64(x[sel])
    out = np.zeros((sel.size, x.shape[1]), dtype=np.float64)
    if "ws1" in inp:
        out += swiglu_expert(xs, inp["ws1"], inp["ws3"], inp["ws2"])
    idx = routing.topk_idx[sel]
    w = routing.topk_w[sel]
    for e in range(inp["w1"].shape[0]):
        rows, cols = np.nonzero(idx == e)          # rows in token order
        if rows.size == 0:
            continue
        y = swiglu_expert(xs[rows], inp["w1"][e], inp["w3"][e], inp["w2"][e])
        np.add.at(out, rows, w[rows, cols][:, None] * y)
    return out, routing


def combine(y_perm, slot_pos, topk_w, y_shared=None) -> np.ndarray:
    """Weighted un-permute: out[t] = y_shared[t] + sum_j w[t, j] * y_perm[slot_pos[t, j]].

    The "weighted sum" of the "Architecture diagram" in the
    "moe-200m-qwen3-100b" README, with the routed outputs held in
    expert-contiguous rows.  Pairs with a negative slot contribute nothing.
    """
    y = _as64(y_perm)
    sp = np.asarray(slot_pos, dtype=np.int64)
    w = _as64(topk_w)
    T, k = sp.shape
    out = np.zeros((T, y.shape[1])) if y_shared is None else _as64(y_shared).copy()
    for j in range(k):
        ok = sp[:, j] >= 0
        out[ok] += w[ok, j:j + 1] * y[sp[ok, j]]
    return out


def moe_forward_dense_masked(inp: dict, top_k: int, gate: int, norm_topk_prob: bool):
    """Brute force: every expert on every token, masked by the combine weights.

    For tiny inputs only.  Builds the dense [T, E] gate matrix holding w[t, j]
    at column idx[t, j] and zero elsewhere, runs all E experts on all tokens and
    sums mask-weighted outputs.  Used to check the routed (sorted) evaluation.
    """
    x = inp["x"]
    r = router(x, inp["w_router"], top_k, gate, norm_topk_prob,
               inp.get("sel_bias"), inp.get("logit_offset"))
    T, E = x.shape[0], inp["w1"].shape[0]
    mask = np.zeros((T, E))
    for t in range(T):
        for j in range(top_k):
            mask[t, r.topk_idx[t, j]] = r.topk_w[t, j]
    out = np.zeros((T, x.shape[1]))
    if "ws1" in inp:
        out += swiglu_expert(x, inp["ws1"], inp["ws3"], inp["ws2"])
    for e in range(E):
        out += mask[:, e:e + 1] * swiglu_expert(x, inp["w1"][e], inp["w3"][e], inp["w2"][e])
    return out


def bias_update(counts, sel_bias, rate: float = 1e-3, starved_frac: float = 0.1,
                starved_add: float = 0.5, clamp: float = 10.0) -> np.ndarray:
    """Aux-loss-free bias controller, one step, in float32.

    ``step_bias_update`` ("moe-200m-qwen3-100b" README, "SigmoidRouter"):
      p_e    = c_e / max(sum c, 1)
      err_e  = 1/E - p_e + starved_add * [p_e < starved_frac / E]
      bias_e = clamp(bias_e + rate * err_e, -clamp, +clamp)
    The bias is an fp32 buffer and counts are converted to fp32 first.  Python
    scalars enter the fp32 arithmetic rounded to fp32: 1/E and starved_frac/E
    are formed in double and then rounded.  Each operation is one fp32
    operation, in the order written (no fused multiply-add).
    """
    f32 = np.float32
    c = np.asarray(counts).astype(f32)
    b = np.asarray(sel_bias, dtype=f32).copy()
    E = c.size
    total = f32(c.sum(dtype=f32))          # integer-valued, exact below 2**24
    total = max(total, f32(1.0))
    p = (c / total).astype(f32)
    target = f32(1.0 / E)
    thresh = f32(starved_frac * (1.0 / E))
    err = (target - p).astype(f32)
    starved = (p < thresh).astype(f32)
    err = (err + (starved * f32(starved_add)).astype(f32)).astype(f32)
    step = (err * f32(rate)).astype(f32)
    b = (b + step).astype(f32)
    b = np.minimum(np.maximum(b, f32(-clamp)), f32(clamp)).astype(f32)
    return b


def bias_update_sign(counts, sel_bias, rate: float = 1e-3) -> np.ndarray:
    """Aux-loss-free bias update of the noaux_tc kind, one micro-batch, float32.

    SpecForge PR #931, "What to watch": with rate 0.001 and 64 accumulation
    steps per optimizer step (its setup) the selection bias "grows linearly
    (0.064/step at this accumulation)", i.e. every micro-batch moves a bias
    by a fixed step toward balance:
        bias_e += rate * sign(mean(c) - c_e)      (sign(0) = 0, no clamp)
    mean(c) = fp32(sum c) / fp32(E), one fp32 operation per step.
    """
    f32 = np.float32
    c = np.asarray(counts).astype(f32)
    b = np.asarray(sel_bias, dtype=f32).copy()
    mean = (f32(c.sum(dtype=f32)) / f32(c.size)).astype(f32)
    d = (mean - c).astype(f32)
    step = np.sign(d).astype(f32) * f32(rate)
    return (b + step.astype(f32)).astype(f32)


def router_stats(routing: Routing) -> dict:
    """Router losses and health metrics, fp64.

    "moe-200m-qwen3-100b" README, SigmoidRouter forward ("ST-MoE z-loss +
    DeepSeek aux loss" and "Routing health metrics"):
      z_loss       = mean_t (logsumexp_e logits[t, e])^2
      aux_loss     = E * sum_e (one_hot.mean over tokens)_e * (scores.mean over tokens)_e
      counts       = one_hot summed over tokens
      cv           = std(counts) / max(mean(counts), 1)   (std with Bessel's correction,
                                                          torch's default)
      entropy_bits = -sum p log p / log 2 with p = max(mean scores, 1e-9), normalised
    and SpecForge PR #931 ("What to watch"): load_max_ratio = max(counts) /
    (mean counts) (ceiling E / k) and the fraction of experts with no tokens.
    """
    lg = routing.logits
    T, E = lg.shape
    m = lg.max(axis=1, keepdims=True)
    lse = (m + np.log(np.exp(lg - m).sum(axis=1, keepdims=True)))[:, 0]
    z_loss = float(np.mean(lse ** 2))
    one_hot = np.zeros((T, E))
    for j in range(routing.topk_idx.shape[1]):
        one_hot[np.arange(T), routing.topk_idx[:, j]] += 1.0
    p = routing.scores.mean(axis=0)
    aux_loss = float(E * np.sum(one_hot.mean(axis=0) * p))
    counts = one_hot.sum(axis=0)
    cv = float(np.std(counts, ddof=1) / max(counts.mean(), 1.0)) if E > 1 else float("nan")
    pa = np.maximum(p, 1e-9)
    pa = pa / pa.sum()
    entropy_bits = float(-np.sum(pa * np.log(pa)) / np.log(2.0))
    mean_c = counts.sum() / E
    load_max_ratio = float(counts.max() / mean_c) if mean_c > 0 else 0.0
    unused = float(np.mean(counts == 0))
    return {"z_loss": z_loss, "aux_loss": aux_loss, "cv": cv, "entropy_bits": entropy_bits,
            "load_max_ratio": load_max_ratio, "unused_frac": unused, "counts": counts}


def _swiglu_expert_backward(xr, w1, w3, w2, dy):
    """Gradients of one SwiGLU expert y = w2 (silu(w1 x) * (w3 x)) on rows xr.

    Chain rule through the three linears and silu, silu'(g) = s(g) (1 + g (1 - s(g)))
    with s the logistic function.  Returns (dx [n, d], dw1 [F, d], dw3 [F, d],
    dw2 [d, F]).
    """
    xr, dy = _as64(xr), _as64(dy)
    w1, w3, w2 = _as64(w1), _as64(w3), _as64(w2)
    g = xr @ w1.T
    u = xr @ w3.T
    sg = sigmoid(g)
    h = g * sg * u                       # silu(g) * u
    dh = dy @ w2                         # [n, F]
    du = dh * (g * sg)                   # d/du of silu(g) u
    dg = dh * u * (sg * (1.0 + g * (1.0 - sg)))
    dx = dg @ w1 + du @ w3
    return dx, dg.T @ xr, du.T @ xr, dy.T @ h


def moe_backward(inp: dict, top_k: int, gate: int, norm_topk_prob: bool, dout,
                 routing: Optional[Routing] = None) -> dict:
    """Gradients of the layer output with respect to x and every weight.

    The layer is the forward of ``moe_forward`` (the pages train it: the
    "moe-200m-qwen3-100b" README trains the SigmoidRouter layer end to end,
    SpecForge PR #930 trains the qwen3 drafter).  Given dout [T, d]:

    * combine: dw[t, j] = <dout[t], y[t, j]>, the expert input gradient is
      w[t, j] dout[t]; the shared expert gets dout[t] with weight 1;
    * experts: the SwiGLU chain rule (``_swiglu_expert_backward``), weight
      gradients summed over the expert's rows;
    * router: the selection (top-k of logits + bias (+ noise)) is piecewise
      constant, so bias and noise get no gradient; the weights are
      w_j = s_j / (sum_i s_i + 1e-9) (or s_j without renormalisation) with
      s = sigmoid(logits) or softmax(logits) over all E, so
      ds_j = (dw_j - sum_i dw_i w_i) / (sum_i s_i + 1e-9) (ds_j = dw_j without
      renormalisation), zero for experts not picked; dlogits =
      ds * s (1 - s) for sigmoid and s * (ds - <ds, s>) for softmax;
      logits = x w_router^T + offset gives dw_router = dlogits^T x and
      dx += dlogits w_router.

    Returns a dict of fp64 arrays: dx, dw_router, dw1, dw3, dw2, dws1, dws3,
    dws2 (the last three only with a shared expert), dlogits, dtopk_w.
    """
    x = _as64(inp["x"])
    dout = _as64(dout)
    T, d = x.shape
    if routing is None:
        routing = router(x, inp["w_router"], top_k, gate, norm_topk_prob,
                         inp.get("sel_bias"), inp.get("logit_offset"))
    idx, w = routing.topk_idx, routing.topk_w
    E = inp["w1"].shape[0]
    dx = np.zeros((T, d))
    dw1 = np.zeros(_as64(inp["w1"]).shape)
    dw3 = np.zeros_like(dw1)
    dw2 = np.zeros(_as64(inp["w2"]).shape)
    dtopk_w = np.zeros((T, top_k))
    for e in range(E):
        rows, cols = np.nonzero(idx == e)
        if rows.size == 0:
            continue
        xr = x[rows]
        y = swiglu_expert(xr, inp["w1"][e], inp["w3"][e], inp["w2"][e])
        dtopk_w[rows, cols] = np.sum(dout[rows] * y, axis=1)
        dy = w[rows, cols][:, None] * dout[rows]
        gx, g1, g3, g2 = _swiglu_expert_backward(xr, inp["w1"][e], inp["w3"][e],
                                                 inp["w2"][e], dy)
        np.add.at(dx, rows, gx)
        dw1[e] += g1
        dw3[e] += g3
        dw2[e] += g2
    out = {"dw1": dw1, "dw3": dw3, "dw2": dw2, "dtopk_w": dtopk_w}
    if "ws1" in inp:
        gx, g1, g3, g2 = _swiglu_expert_backward(x, inp["ws1"], inp["ws3"], inp["ws2"], dout)
        dx += gx
        out.update(dws1=g1, dws3=g3, dws2=g2)
    # router
    s = routing.scores
    ds = np.zeros((T, E))
    rr = np.arange(T)[:, None]
    if norm_topk_prob:
        ssel = np.take_along_axis(s, idx, axis=1)
        denom = ssel.sum(axis=1, keepdims=True) + 1e-9
        ds[rr, idx] = (dtopk_w - np.sum(dtopk_w * w, axis=1, keepdims=True)) / denom
    else:
        ds[rr, idx] = dtopk_w
    if gate == GATE_SIGMOID:
        dlogits = ds * s * (1.0 - s)
    else:
        dlogits = s * (ds - np.sum(ds * s, axis=1, keepdims=True))
    out["dlogits"] = dlogits
    out["dw_router"] = dlogits.T @ x
    dx += dlogits @ _as64(inp["w_router"])
    out["dx"] = dx
    return out
