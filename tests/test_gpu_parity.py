"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Small shapes span several tiles with ragged tails and are compared element by
element.  The full workload sizes (the ones the benchmark times, in the same
launch configuration) are compared on every routing decision, on the
forward's own permutation (counts, offsets, slots and row order, bit for
bit) and on every output element.
"""
import json
import os

import numpy as np
import pytest
import torch

import _parity as P
from mixture_experts_ffn_bias_b200 import binding as B
from mixture_experts_ffn_bias_b200 import build as build_mod
from mixture_experts_ffn_bias_b200 import inputs as I
from mixture_experts_ffn_bias_b200.layer import MoELayer, to_device
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny": I.WORKLOADS["tiny"],
    "page2_small": I.WORKLOADS["page2"].replace(T=640),
    "qwen3_small": I.WORKLOADS["qwen3_30b"].replace(T=600, d_model=256, d_ff=256),
    "wide_small": I.WORKLOADS["wide"].replace(T=200, d_model=512, d_ff=384),
    "skew_small": I.WORKLOADS["skew"].replace(T=1000, d_model=256, d_ff=256, d_ff_shared=256),
}
FULL = ["page2", "qwen3_30b", "wide", "skew"]
NEAR_TIES = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "near_ties.json")


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build_mod.build()
    B.lib()


def _np(t):
    return t.detach().float().cpu().numpy() if t.dtype == torch.bfloat16 else t.detach().cpu().numpy()


def _tol(shape):
    return P.OUT_TOL_BF16 if shape.dtype == I.DTYPE_BF16 else P.OUT_TOL_F32


def _run(shape, host):
    layer = MoELayer(shape, host)
    layer.forward()
    torch.cuda.synchronize()
    st, flags = layer.device_status()
    assert st == B.MOE_OK, (st, flags)
    return layer


def _check_layer(shape, host, layer, tokens=None, dispatch=True):
    """Routing, counts, the forward's own permutation and the outputs of
    `tokens` (all tokens when None) against the oracle."""
    r = P.oracle_routing(shape, host)
    gidx, gw = _np(layer.topk_idx), _np(layer.topk_w)
    excluded, ordered = P.check_routing(gidx, gw, r)
    P.record_exclusions(shape, excluded, ordered)
    P.check_counts_vs_oracle(_np(layer.counts), r, gidx, shape.n_experts, excluded)
    if dispatch:
        offs, slot, src = (_np(t) for t in layer.dispatch_view())
        P.check_dispatch(gidx, _np(layer.counts), offs, slot, src, r, shape.n_experts, excluded)
    sel = np.arange(shape.T) if tokens is None else tokens
    sel = sel[~excluded[sel]]
    out = _np(layer.out)
    diff = scale = 0.0
    # the oracle in windows of tokens (bounded host memory at full size)
    for lo in range(0, sel.size, 8192):
        part = sel[lo:lo + 8192]
        ref, _ = O.moe_forward(host, shape.top_k, shape.gate, bool(shape.norm_topk_prob),
                               tokens=part, routing=r)
        diff = max(diff, P.abs_err(out[part], ref))
        scale = max(scale, float(np.max(np.abs(ref))))
    err = diff / scale if scale > 0 else diff
    assert err <= _tol(shape), f"output relative error {err:.3e}"
    return r, excluded, err


# --------------------------------------------------------------------------- #
# whole layer                                                                 #
# --------------------------------------------------------------------------- #
@pytest.mark.parametrize("name", list(SMALL))
def test_forward_small_elementwise(name):
    shape = SMALL[name]
    host = I.make_inputs(shape)
    layer = _run(shape, host)
    _check_layer(shape, host, layer)


@pytest.mark.parametrize("name", FULL)
def test_forward_full_size_every_token(name):
    """The benchmark's workloads at full size: every token's experts and
    weights, the per-expert counts, the forward's own permutation bit for
    bit, and every element of the output.  The near-tie exclusions the
    oracle finds must be the ones stored by the oracle-only script
    tests/golden/make_near_ties.py (they are reported at the end of the
    run)."""
    shape = I.WORKLOADS[name]
    host = I.make_inputs(shape)
    layer = _run(shape, host)
    _, excluded, _ = _check_layer(shape, host, layer)
    with open(NEAR_TIES) as f:
        stored = json.load(f)["workloads"][name]
    assert int(excluded.sum()) == stored["excluded"]
    assert excluded.nonzero()[0].tolist() == stored["tokens"]
    del layer
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name", ["page2_small", "qwen3_small", "skew_small", "qwen3_30b"])
def test_forward_with_gathered_gate_up_rows(name):
    """The alternative expert path (moe_forward_ex, gather_rows = 1) that
    skips the permuted copy of x and gathers the gate/up GEMM's rows from x
    (small shapes, and the full qwen3_30b workload on every token)."""
    shape = SMALL[name] if name in SMALL else I.WORKLOADS[name]
    host = I.make_inputs(shape)
    layer = MoELayer(shape, host)
    layer.forward(gather_rows=True)
    torch.cuda.synchronize()
    assert layer.device_status()[0] == B.MOE_OK
    _check_layer(shape, host, layer)


@pytest.mark.parametrize("name,gather", [("page2_small", False), ("qwen3_small", False),
                                         ("skew_small", True), ("qwen3_30b", False),
                                         ("skew", False)])
def test_forward_with_folded_combine(name, gather):
    """The alternative (moe_forward_ex, fold_combine = 1) whose down GEMM
    forms the combined output: against the oracle, and bit for bit against
    the default path's separate combine (the same fp32 operations in the same
    order).  page2_small's d = 640 ends in a half-empty 256-column tile; skew
    has experts that no token chose."""
    shape = SMALL[name] if name in SMALL else I.WORKLOADS[name]
    host = I.make_inputs(shape)
    layer = MoELayer(shape, host)
    layer.forward()
    torch.cuda.synchronize()
    ref = layer.out.clone()
    layer.out.fill_(float("nan"))
    layer.forward(gather_rows=gather, fold_combine=True)
    torch.cuda.synchronize()
    assert layer.device_status()[0] == B.MOE_OK
    assert torch.equal(layer.out.view(torch.int16), ref.view(torch.int16))
    _check_layer(shape, host, layer)


@pytest.mark.parametrize("name,fold", [("page2_small", False), ("qwen3_small", False),
                                       ("skew_small", True), ("wide_small", False),
                                       ("qwen3_30b", False), ("skew", False), ("page2", True)])
def test_forward_with_scatter_in_gemm(name, fold):
    """The alternative (moe_forward_ex, scatter_in_gemm = 1) whose gate/up
    GEMM copies x's rows into x_perm while it runs: against the oracle and
    bit for bit against the default path, with the device status clear (no
    wait gave up).  The backward tests read that x_perm too."""
    shape = SMALL[name] if name in SMALL else I.WORKLOADS[name]
    host = I.make_inputs(shape)
    layer = MoELayer(shape, host)
    layer.forward()
    torch.cuda.synchronize()
    ref = layer.out.clone()
    layer.out.fill_(float("nan"))
    layer.forward(scatter_in_gemm=True, fold_combine=fold)
    torch.cuda.synchronize()
    assert layer.device_status()[0] == B.MOE_OK
    assert torch.equal(layer.out.view(torch.int16), ref.view(torch.int16))
    _check_layer(shape, host, layer)


def test_skew_bias_update_then_deferred_forward():
    """Skewed workload: forward, bias update from its counts (bit-exact), then a
    second forward routes with the new bias (the update lands on the next
    forward)."""
    shape = I.WORKLOADS["skew"].replace(T=4096, d_model=512, d_ff=256, d_ff_shared=256)
    host = I.make_inputs(shape)
    layer = _run(shape, host)
    r = P.oracle_routing(shape, host)
    excluded, _ = P.check_routing(_np(layer.topk_idx), _np(layer.topk_w), r)
    assert not excluded.any()
    counts_ref = O.dispatch(r.topk_idx, shape.n_experts).counts
    np.testing.assert_array_equal(_np(layer.counts), counts_ref)
    assert (counts_ref == 0).any(), "Zipf offsets should starve some experts"
    layer.bias_update(rate=1e-3, starved_frac=0.1, starved_add=0.5, clamp=10.0)
    torch.cuda.synchronize()
    bias_ref = O.bias_update(counts_ref, host["sel_bias"], 1e-3, 0.1, 0.5, 10.0)
    np.testing.assert_array_equal(_np(layer.sel_bias), bias_ref)
    layer.forward()
    torch.cuda.synchronize()
    r2 = P.oracle_routing(shape, host, sel_bias=bias_ref)
    P.check_routing(_np(layer.topk_idx), _np(layer.topk_w), r2)


# --------------------------------------------------------------------------- #
# edge cases                                                                  #
# --------------------------------------------------------------------------- #
def test_single_token():
    shape = SMALL["qwen3_small"].replace(T=1)
    host = I.make_inputs(shape)
    _check_layer(shape, host, _run(shape, host))


def test_zero_tokens_is_a_noop():
    shape = SMALL["page2_small"].replace(T=0)
    cfg = B.config_from_shape(shape)
    counts = torch.full((shape.n_experts,), 7, dtype=torch.int32, device="cuda")
    dummy = torch.empty(64, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    w = {"w1": dummy, "w3": dummy, "w2": dummy, "ws1": dummy, "ws3": dummy, "ws2": dummy}
    assert B.moe_forward(cfg, dummy, dummy, None, None, w, dummy, dummy, dummy, counts, ws) == 0
    torch.cuda.synchronize()
    assert int(counts.abs().sum()) == 0


def test_large_experts_use_m_fastest_tile_order():
    """Experts whose weights exceed a quarter of L2 are tiled m-fastest; check
    that order element-wise (two 5120 x 4352 experts, ragged rows)."""
    shape = I.MoEShape("big_experts", 333, 5120, 2, 4352, 1, 0, 0, I.GATE_SOFTMAX, 1,
                       I.DTYPE_BF16, "uniform", 0.0, 10)
    host = I.make_inputs(shape)
    _check_layer(shape, host, _run(shape, host))


def test_one_expert_top1_is_dense_ffn():
    shape = I.MoEShape("one", 300, 256, 1, 256, 1, 0, 0, I.GATE_SOFTMAX, 1, I.DTYPE_BF16,
                       "none", 0.0, 7)
    host = I.make_inputs(shape)
    _check_layer(shape, host, _run(shape, host))


def test_top_k_equals_all_experts():
    shape = I.MoEShape("all", 257, 128, 8, 128, 8, 0, 0, I.GATE_SOFTMAX, 1, I.DTYPE_BF16,
                       "none", 0.0, 8)
    host = I.make_inputs(shape)
    _check_layer(shape, host, _run(shape, host))


def test_every_token_on_one_expert():
    """A huge bias on one expert: one segment of T rows, all others empty."""
    shape = SMALL["skew_small"].replace(T=700)
    host = I.make_inputs(shape)
    host["sel_bias"] = np.zeros(shape.n_experts, np.float32)
    host["sel_bias"][37] = 50.0
    layer = _run(shape, host)
    c = _np(layer.counts)
    assert c[37] == shape.T and c.sum() == shape.T * shape.top_k
    _check_layer(shape, host, layer)


def _edge_shape(name):
    if name == "single_token":
        return SMALL["qwen3_small"].replace(T=1), None
    if name == "one_expert_top1":
        return I.MoEShape("one", 300, 256, 1, 256, 1, 0, 0, I.GATE_SOFTMAX, 1, I.DTYPE_BF16,
                          "none", 0.0, 7), None
    if name == "top_k_all":
        return I.MoEShape("all", 257, 128, 8, 128, 8, 0, 0, I.GATE_SOFTMAX, 1, I.DTYPE_BF16,
                          "none", 0.0, 8), None
    bias = np.zeros(64, np.float32)   # every token on expert 37, with a shared expert
    bias[37] = 50.0
    return SMALL["skew_small"].replace(T=700), bias


@pytest.mark.parametrize("name", ["single_token", "one_expert_top1", "top_k_all", "one_hot"])
@pytest.mark.parametrize("opt", ["fold_combine", "scatter_in_gemm", "gather_rows"])
def test_forward_options_on_edge_shapes(name, opt):
    """Each per-call alternative on the degenerate shapes (one token; one
    expert, top-1; top-k = E; every token on one expert next to 63 empty
    ones and a shared expert): bit for bit against the default path and
    element-wise against the oracle."""
    shape, bias = _edge_shape(name)
    host = I.make_inputs(shape)
    if bias is not None:
        host["sel_bias"] = bias
    layer = MoELayer(shape, host)
    layer.forward()
    torch.cuda.synchronize()
    ref = layer.out.clone()
    layer.out.fill_(float("nan"))
    layer.forward(**{opt: True})
    torch.cuda.synchronize()
    assert layer.device_status()[0] == B.MOE_OK
    assert torch.equal(layer.out.view(torch.int16), ref.view(torch.int16))
    _check_layer(shape, host, layer)


@pytest.mark.parametrize("E,k,gate", [(256, 4, I.GATE_SOFTMAX), (32, 12, I.GATE_SIGMOID),
                                      (200, 3, I.GATE_SIGMOID)])
def test_router_paths_without_fused_select(E, k, gate):
    """More than 128 experts or top-k above 8: logits are written out and a
    separate selection kernel decides."""
    shape = I.MoEShape("unfused", 300, 256, E, 128, k, 0, 0, gate, 1, I.DTYPE_BF16,
                       "uniform", 0.0, 9)
    host = I.make_inputs(shape)
    _check_layer(shape, host, _run(shape, host))


@pytest.mark.parametrize("gate", [I.GATE_SOFTMAX, I.GATE_SIGMOID])
def test_exact_key_ties_are_redecided_to_the_lower_expert(gate):
    """Two experts with identical router rows and bias tie exactly on every
    token; those tokens go through the exact re-decision, which must pick the
    lower expert id first, as the oracle does."""
    shape = SMALL["qwen3_small"].replace(T=400, gate=gate)
    host = I.make_inputs(shape)
    host["w_router"][77] = host["w_router"][5]
    host["sel_bias"] = np.zeros(shape.n_experts, np.float32)
    layer = _run(shape, host)
    r = P.oracle_routing(shape, host)
    gidx = _np(layer.topk_idx)
    both = np.isin(r.topk_idx, [5, 77]).sum(1) == 2
    assert both.any()
    _check_layer(shape, host, layer)
    np.testing.assert_array_equal(gidx[both], r.topk_idx[both])


@pytest.mark.parametrize("gate", [I.GATE_SOFTMAX, I.GATE_SIGMOID])
def test_constant_bias_moves_nothing_on_gpu(gate):
    shape = SMALL["qwen3_small"].replace(gate=gate, T=512)
    host = I.make_inputs(shape)
    a = _run(shape, host)
    idx0, w0 = _np(a.topk_idx).copy(), _np(a.topk_w).copy()
    host2 = dict(host)
    host2["sel_bias"] = np.full(shape.n_experts, 0.25, np.float32)
    b = _run(shape, host2)
    np.testing.assert_array_equal(_np(b.topk_idx), idx0)
    np.testing.assert_array_equal(_np(b.topk_w), w0)


# --------------------------------------------------------------------------- #
# the individual calls                                                        #
# --------------------------------------------------------------------------- #
def _buffers(shape):
    cfg = B.config_from_shape(shape)
    ws = torch.empty(B.moe_workspace_size(cfg), dtype=torch.uint8, device="cuda")
    return cfg, ws


@pytest.mark.parametrize("name", ["tiny", "page2_small", "skew_small"])
def test_router_topk_call(name):
    shape = SMALL[name]
    host = I.make_inputs(shape)
    cfg, ws = _buffers(shape)
    dt = torch.bfloat16 if shape.dtype == I.DTYPE_BF16 else torch.float32
    x = to_device(host["x"], dt, "cuda")
    wr = to_device(host["w_router"], dt, "cuda")
    bias = to_device(host["sel_bias"], torch.float32, "cuda") if "sel_bias" in host else None
    off = (to_device(host["logit_offset"], torch.float32, "cuda")
           if "logit_offset" in host else None)
    idx = torch.empty((shape.T, shape.top_k), dtype=torch.int32, device="cuda")
    w = torch.empty((shape.T, shape.top_k), dtype=torch.float32, device="cuda")
    B.moe_router_topk(cfg, x, wr, bias, off, idx, w, ws)
    torch.cuda.synchronize()
    P.check_routing(_np(idx), _np(w), P.oracle_routing(shape, host))


@pytest.mark.parametrize("name", ["tiny", "page2_small", "qwen3_small", "skew_small"])
@pytest.mark.parametrize("space,noisy", [(1, False), (0, True), (1, True)])
def test_router_key_variants_call(name, space, noisy):
    """moe_router_topk_opts: bias on the gate scores and/or a given
    selection noise [T, E], against the oracle's router with the same
    options; the weights stay the unbiased scores."""
    shape = SMALL[name]
    host = I.make_inputs(shape)
    if "sel_bias" not in host:
        host["sel_bias"] = np.random.default_rng(31).uniform(
            -0.05, 0.05, shape.n_experts).astype(np.float32)
    cfg, ws = _buffers(shape)
    dt = torch.bfloat16 if shape.dtype == I.DTYPE_BF16 else torch.float32
    x = to_device(host["x"], dt, "cuda")
    wr = to_device(host["w_router"], dt, "cuda")
    bias = to_device(host["sel_bias"], torch.float32, "cuda")
    off = (to_device(host["logit_offset"], torch.float32, "cuda")
           if "logit_offset" in host else None)
    noise = None
    if noisy:
        noise = (0.1 * np.random.default_rng(32).standard_normal(
            (shape.T, shape.n_experts))).astype(np.float32)
    idx = torch.empty((shape.T, shape.top_k), dtype=torch.int32, device="cuda")
    w = torch.empty((shape.T, shape.top_k), dtype=torch.float32, device="cuda")
    B.moe_router_topk_opts(cfg, x, wr, bias, off, idx, w, ws, bias_space=space,
                           sel_noise=None if noise is None else to_device(noise, torch.float32,
                                                                          "cuda"))
    torch.cuda.synchronize()
    r = O.router(host["x"], host["w_router"], shape.top_k, shape.gate,
                 bool(shape.norm_topk_prob), host["sel_bias"], host.get("logit_offset"),
                 bias_space=space, sel_noise=noise)
    P.check_routing(_np(idx), _np(w), r)


def test_router_opts_default_is_router_topk():
    shape = SMALL["qwen3_small"]
    host = I.make_inputs(shape)
    cfg, ws = _buffers(shape)
    x = to_device(host["x"], torch.bfloat16, "cuda")
    wr = to_device(host["w_router"], torch.bfloat16, "cuda")
    out = []
    for opts in (False, True):
        idx = torch.empty((shape.T, shape.top_k), dtype=torch.int32, device="cuda")
        w = torch.empty((shape.T, shape.top_k), dtype=torch.float32, device="cuda")
        if opts:
            B.moe_router_topk_opts(cfg, x, wr, None, None, idx, w, ws)
        else:
            B.moe_router_topk(cfg, x, wr, None, None, idx, w, ws)
        torch.cuda.synchronize()
        out.append((_np(idx), _np(w)))
    np.testing.assert_array_equal(out[0][0], out[1][0])
    np.testing.assert_array_equal(out[0][1], out[1][1])


@pytest.mark.parametrize("name", FULL)
def test_tensor_core_logit_error_is_far_below_the_refine_margin(name):
    """The router decides from tensor-core fp32 logits and re-decides on exact
    logits any token whose keys lie within 1e-4 of each other.  That is only
    sound if the fp32 logits are much closer than 1e-4 to the exact ones;
    measure it on every logit of the full workload."""
    shape = I.WORKLOADS[name]
    rng_host = I.make_inputs(shape)
    cfg, ws = _buffers(shape)
    x = to_device(rng_host["x"], torch.bfloat16, "cuda")
    wr = to_device(rng_host["w_router"], torch.bfloat16, "cuda")
    logits = torch.empty((shape.T, shape.n_experts), dtype=torch.float32, device="cuda")
    B.moe_router_logits(cfg, x, wr, None, logits, ws)
    torch.cuda.synchronize()
    exact = rng_host["x"].astype(np.float64) @ rng_host["w_router"].astype(np.float64).T
    err = float(np.max(np.abs(_np(logits) - exact)))
    assert err < 5e-6, f"max |fp32 tensor-core logit - exact| = {err:.3e}"


@pytest.mark.parametrize("name", ["tiny", "qwen3_small", "skew_small"])
def test_permute_call_bit_exact(name):
    """Oracle routing in, dispatch out: counts, offsets, slots, rows bit-exact."""
    shape = SMALL[name]
    host = I.make_inputs(shape)
    r = P.oracle_routing(shape, host)
    ref = O.dispatch(r.topk_idx, shape.n_experts)
    cfg, ws = _buffers(shape)
    dt = torch.bfloat16 if shape.dtype == I.DTYPE_BF16 else torch.float32
    T, k, E, d = shape.T, shape.top_k, shape.n_experts, shape.d_model
    x = to_device(host["x"], dt, "cuda")
    idx = torch.from_numpy(r.topk_idx.astype(np.int32)).cuda()
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    slot = torch.empty((T, k), dtype=torch.int32, device="cuda")
    src = torch.empty(T * k, dtype=torch.int32, device="cuda")
    xp = torch.empty((T * k, d), dtype=dt, device="cuda")
    B.moe_permute(cfg, idx, x, counts, offsets, slot, src, xp, ws)
    assert B.moe_device_status(ws)[0] == B.MOE_OK
    np.testing.assert_array_equal(_np(counts), ref.counts)
    np.testing.assert_array_equal(_np(offsets), ref.offsets)
    np.testing.assert_array_equal(_np(slot), ref.slot_pos)
    np.testing.assert_array_equal(_np(src), ref.perm_src)
    np.testing.assert_array_equal(_np(xp), host["x"][ref.perm_src])


def test_permute_skips_and_reports_bad_ids():
    shape = SMALL["qwen3_small"].replace(T=300)
    host = I.make_inputs(shape)
    r = P.oracle_routing(shape, host)
    bad = r.topk_idx.astype(np.int32).copy()
    bad[5, 2] = -3                       # out of range
    bad[17, 0] = shape.n_experts         # out of range
    bad[40, 3] = bad[40, 1]              # repeated within the token
    cfg, ws = _buffers(shape)
    T, k, E, d = shape.T, shape.top_k, shape.n_experts, shape.d_model
    x = to_device(host["x"], torch.bfloat16, "cuda")
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    slot = torch.empty((T, k), dtype=torch.int32, device="cuda")
    src = torch.empty(T * k, dtype=torch.int32, device="cuda")
    xp = torch.empty((T * k, d), dtype=torch.bfloat16, device="cuda")
    B.moe_permute(cfg, torch.from_numpy(bad).cuda(), x, counts, offsets, slot, src, xp, ws)
    st, flags = B.moe_device_status(ws)
    assert st == B.MOE_ERR_DATA and flags & 1
    s = _np(slot)
    assert s[5, 2] == -1 and s[17, 0] == -1 and s[40, 3] == -1
    valid = s >= 0
    assert int(_np(offsets)[-1]) == valid.sum() == T * k - 3
    # the valid pairs keep the stable (expert, token) order
    e_of = bad.reshape(-1)[valid.reshape(-1)]
    t_of = np.repeat(np.arange(T), k)[valid.reshape(-1)]
    order = np.lexsort((t_of, e_of))
    np.testing.assert_array_equal(np.sort(s[valid]), np.arange(valid.sum()))
    np.testing.assert_array_equal(s.reshape(-1)[valid.reshape(-1)][order], np.arange(valid.sum()))


@pytest.mark.parametrize("name", ["tiny", "page2_small", "wide_small"])
def test_grouped_swiglu_call(name):
    """Oracle dispatch in; every expert row against the oracle's expert."""
    shape = SMALL[name]
    host = I.make_inputs(shape)
    r = P.oracle_routing(shape, host)
    dp = O.dispatch(r.topk_idx, shape.n_experts)
    cfg, ws = _buffers(shape)
    dt = torch.bfloat16 if shape.dtype == I.DTYPE_BF16 else torch.float32
    T, k, d = shape.T, shape.top_k, shape.d_model
    xp = to_device(host["x"][dp.perm_src], dt, "cuda")
    offs = torch.from_numpy(dp.offsets.astype(np.int32)).cuda()
    wts = {key: to_device(host[key], dt, "cuda") for key in ("w1", "w3", "w2", "ws1", "ws3", "ws2")
           if key in host}
    x = to_device(host["x"], dt, "cuda")
    yp = torch.empty((T * k, d), dtype=dt, device="cuda")
    ysh = torch.empty((T, d), dtype=dt, device="cuda") if shape.n_shared else None
    B.moe_grouped_swiglu(cfg, xp, offs, wts, x if shape.n_shared else None, yp, ysh, ws)
    assert B.moe_device_status(ws)[0] == B.MOE_OK
    ref = np.concatenate([
        O.swiglu_expert(host["x"][dp.perm_src[dp.offsets[e]:dp.offsets[e + 1]]],
                        host["w1"][e], host["w3"][e], host["w2"][e])
        for e in range(shape.n_experts)])
    assert P.rel_err(_np(yp), ref) <= _tol(shape)
    if shape.n_shared:
        ref_sh = O.swiglu_expert(host["x"], host["ws1"], host["ws3"], host["ws2"])
        assert P.rel_err(_np(ysh), ref_sh) <= _tol(shape)


@pytest.mark.parametrize("bf16,shared", [(True, True), (True, False), (False, False)])
def test_combine_call(bf16, shared):
    rng = np.random.default_rng(5)
    T, k, d = 333, 3, 256
    R = T * k
    dt = torch.bfloat16 if bf16 else torch.float32
    y = I.round_to_bf16(rng.standard_normal((R, d)).astype(np.float32)) if bf16 else \
        rng.standard_normal((R, d)).astype(np.float32)
    ysh = I.round_to_bf16(rng.standard_normal((T, d)).astype(np.float32)) if shared else None
    slot = rng.permutation(R).reshape(T, k).astype(np.int32)
    slot[7, 1] = -1
    w = rng.uniform(0, 1, (T, k)).astype(np.float32)
    cfg = B.make_config(T, d, 8, 128, k, 1 if shared else 0, 128,
                        dtype=B.DTYPE_BF16 if bf16 else B.DTYPE_F32)
    out = torch.empty((T, d), dtype=dt, device="cuda")
    B.moe_combine(cfg, to_device(y, dt, "cuda"), torch.from_numpy(slot).cuda(),
                  torch.from_numpy(w).cuda(), to_device(ysh, dt, "cuda") if shared else None, out)
    torch.cuda.synchronize()
    ref = O.combine(y, slot, w, ysh)
    assert P.rel_err(_np(out), ref) <= (4e-3 if bf16 else 1e-6)


@pytest.mark.parametrize("E", [4, 16, 64, 128])
def test_bias_update_call_bit_exact(E):
    rng = np.random.default_rng(E)
    for trial in range(4):
        counts = rng.integers(0, 3000, E).astype(np.int32)
        counts[rng.integers(0, E, 2)] = 0
        bias = rng.uniform(-9.99, 9.99, E).astype(np.float32)
        if trial == 3:
            bias[:] = 9.9995   # saturation path
        cfg = B.make_config(16, 128, E, 128, 1)
        c_d = torch.from_numpy(counts).cuda()
        b_d = torch.from_numpy(bias.copy()).cuda()
        rate = [1e-3, 0.37, 1e-3, 1.0][trial]
        B.moe_bias_update(cfg, c_d, b_d, rate, 0.1, 0.5, 10.0)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(_np(b_d), O.bias_update(counts, bias, rate, 0.1, 0.5, 10.0))


@pytest.mark.parametrize("E", [16, 64, 128])
def test_bias_update_sign_call_bit_exact(E):
    """noaux_tc-style update: 64 calls on the GPU equal 64 oracle steps bitwise."""
    rng = np.random.default_rng(100 + E)
    counts = rng.integers(0, 900, E).astype(np.int32)
    counts[:3] = [0, int(counts.mean()), 5000]
    cfg = B.make_config(16, 128, E, 128, 1)
    bias = rng.uniform(-1, 1, E).astype(np.float32)
    c_d = torch.from_numpy(counts).cuda()
    b_d = torch.from_numpy(bias.copy()).cuda()
    ref = bias.copy()
    for _ in range(64):
        B.moe_bias_update_sign(cfg, c_d, b_d, 1e-3)
        ref = O.bias_update_sign(counts, ref, 1e-3)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(_np(b_d), ref)


@pytest.mark.parametrize("name", ["tiny", "page2_small", "qwen3_small", "skew_small"])
def test_router_stats_call(name):
    """Router losses and health metrics on the GPU vs the oracle (same routing)."""
    shape = SMALL[name]
    host = I.make_inputs(shape)
    r = P.oracle_routing(shape, host)
    cfg, ws = _buffers(shape)
    dt = torch.bfloat16 if shape.dtype == I.DTYPE_BF16 else torch.float32
    x = to_device(host["x"], dt, "cuda")
    wr = to_device(host["w_router"], dt, "cuda")
    off = (to_device(host["logit_offset"], torch.float32, "cuda")
           if "logit_offset" in host else None)
    idx = torch.from_numpy(r.topk_idx.astype(np.int32)).cuda()
    stats = torch.zeros(8, dtype=torch.float32, device="cuda")
    B.moe_router_stats(cfg, x, wr, off, idx, stats, ws)
    got = _np(stats)
    ref = O.router_stats(r)
    for i, key in enumerate(B.STAT_NAMES):
        assert abs(got[i] - ref[key]) <= 1e-5 * max(1.0, abs(ref[key])), (key, got[i], ref[key])


def test_bounded_wait_gives_up_and_reports_timeout():
    """A wait on a barrier nothing completes runs out after 50 ms; the host
    reads MOE_ERR_TIMEOUT from the status word and the context still works."""
    ws = torch.empty(4096, dtype=torch.uint8, device="cuda")
    B.moe_selftest_bounded_wait(ws, 0.05)
    st, flags = B.moe_device_status(ws)
    assert st == B.MOE_ERR_TIMEOUT and flags & 2
    assert B.moe_device_status(ws)[0] == B.MOE_OK      # read clears the word
    shape = SMALL["qwen3_small"].replace(T=64)
    host = I.make_inputs(shape)
    _check_layer(shape, host, _run(shape, host))


@pytest.mark.parametrize("name", ["qwen3_small", "skew_small"])
def test_token_sharded_routing_equals_whole_batch(name):
    """Data-parallel replicas route their own token shards: every token's
    experts and weights must equal those of the single-GPU run bit for bit
    (the page-2 DDP-vs-single-GPU parity check).  Shards are cut at a
    position that is not a multiple of the 128-token router tile."""
    shape = SMALL[name]
    host = I.make_inputs(shape)
    full = _run(shape, host)
    cut = shape.T // 3 + 5
    parts = []
    for lo, hi in ((0, cut), (cut, shape.T)):
        h = dict(host)
        h["x"] = host["x"][lo:hi]
        sub = _run(shape.replace(T=hi - lo), h)
        parts.append((_np(sub.topk_idx), _np(sub.topk_w)))
    np.testing.assert_array_equal(np.concatenate([p[0] for p in parts]), _np(full.topk_idx))
    np.testing.assert_array_equal(np.concatenate([p[1] for p in parts]), _np(full.topk_w))
