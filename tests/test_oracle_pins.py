"""Pins for the CPU oracle: it is checked against what the pages and the
mathematics fix, never against itself.

Each test names the mistake it would catch.  Sources: "moe-200m-qwen3-100b"
README (SigmoidRouter, step_bias_update, architecture diagram), SpecForge PR
#930 (qwen3 preset, tests, activated-width invariant) and PR #931 (load ceiling,
per-expert keys, grouped GEMM vs sorted loop).
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special

from oracle import moe_oracle as O
from mixture_experts_ffn_bias_b200 import inputs as I

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _ev(v):
    if isinstance(v, str):
        return float(eval(v, {"__builtins__": {}}, {"ln": math.log}))
    return float(v)


def _arr(a):
    if isinstance(a, list):
        return np.array([_arr(v) for v in a], dtype=np.float64)
    return _ev(a)


def _gate(name):
    return O.GATE_SOFTMAX if name == "softmax" else O.GATE_SIGMOID


@pytest.fixture(scope="module")
def worked():
    with open(os.path.join(GOLDEN, "worked_examples.json")) as f:
        return json.load(f)


@pytest.fixture(scope="module")
def figures():
    with open(os.path.join(GOLDEN, "page_figures.json")) as f:
        return json.load(f)


def _random_layer(rng, T, d, E, F, k, shared=False, bias=False, offset=False):
    inp = {
        "x": rng.standard_normal((T, d)),
        "w_router": 0.3 * rng.standard_normal((E, d)),
        "w1": 0.3 * rng.standard_normal((E, F, d)),
        "w3": 0.3 * rng.standard_normal((E, F, d)),
        "w2": 0.3 * rng.standard_normal((E, d, F)),
    }
    if shared:
        inp["ws1"] = 0.3 * rng.standard_normal((F, d))
        inp["ws3"] = 0.3 * rng.standard_normal((F, d))
        inp["ws2"] = 0.3 * rng.standard_normal((d, F))
    if bias:
        inp["sel_bias"] = rng.uniform(-0.5, 0.5, E)
    if offset:
        inp["logit_offset"] = rng.uniform(-1, 1, E)
    return inp


# --------------------------------------------------------------------------- #
# worked examples (closed forms)                                              #
# --------------------------------------------------------------------------- #
def test_worked_softmax_router(worked):
    """Catches: softmax over the wrong axis, missing renorm, wrong top-k order."""
    c = worked["softmax_top2_renorm"]
    r = O.router(_arr(c["x"]), _arr(c["w_router"]), c["top_k"], _gate(c["gate"]),
                 c["norm_topk_prob"])
    np.testing.assert_allclose(r.scores, _arr(c["expected_scores"]), rtol=0, atol=1e-15)
    assert r.topk_idx.tolist() == c["expected_idx"]
    np.testing.assert_allclose(r.topk_w, _arr(c["expected_w"]), rtol=0, atol=1e-15)


def test_worked_sigmoid_bias_moves_selection_only(worked):
    """Catches: bias added to the scores used as weights, or not used for selection."""
    c = worked["sigmoid_bias_moves_selection_only"]
    x, w = _arr(c["x"]), _arr(c["w_router"])
    r0 = O.router(x, w, c["top_k"], _gate(c["gate"]), c["norm_topk_prob"])
    np.testing.assert_allclose(r0.scores, _arr(c["expected_scores"]), rtol=0, atol=1e-15)
    assert r0.topk_idx.tolist() == c["without_bias"]["expected_idx"]
    np.testing.assert_allclose(r0.topk_w, _arr(c["without_bias"]["expected_w"]), atol=1e-15)
    r1 = O.router(x, w, c["top_k"], _gate(c["gate"]), c["norm_topk_prob"],
                  sel_bias=np.array(c["sel_bias"]))
    assert r1.topk_idx.tolist() == c["with_bias"]["expected_idx"]
    np.testing.assert_allclose(r1.topk_w, _arr(c["with_bias"]["expected_w"]), atol=1e-15)
    np.testing.assert_array_equal(r1.scores, r0.scores)


def test_worked_layer_output(worked):
    """Catches: gate/up/down roles swapped, shared expert dropped or weighted."""
    c = worked["layer_single_expert_with_shared"]
    inp = {k: _arr(c[k]) for k in ("x", "w_router", "w1", "w3", "w2", "ws1", "ws3", "ws2")}
    out, r = O.moe_forward(inp, c["top_k"], _gate(c["gate"]), c["norm_topk_prob"])
    assert r.topk_idx.tolist() == c["expected_idx"]
    np.testing.assert_allclose(r.topk_w, _arr(c["expected_w"]), atol=1e-15)
    np.testing.assert_allclose(out, _arr(c["expected_out"]), rtol=1e-14, atol=1e-14)


# --------------------------------------------------------------------------- #
# router invariants                                                           #
# --------------------------------------------------------------------------- #
@pytest.mark.parametrize("gate", [O.GATE_SOFTMAX, O.GATE_SIGMOID])
def test_renormalised_weights_sum_to_one(gate):
    """SpecForge PR #930 'Tests': top-k weights renormalise to one."""
    rng = np.random.default_rng(1)
    inp = _random_layer(rng, 500, 24, 16, 4, 4, bias=True)
    r = O.router(inp["x"], inp["w_router"], 4, gate, True, inp["sel_bias"])
    assert np.max(np.abs(r.topk_w.sum(1) - 1.0)) <= 1e-6


@pytest.mark.parametrize("gate", [O.GATE_SOFTMAX, O.GATE_SIGMOID])
def test_constant_bias_changes_nothing(gate):
    """A bias equal on every expert moves no selection: idx and w identical."""
    rng = np.random.default_rng(2)
    inp = _random_layer(rng, 300, 16, 12, 4, 3)
    r0 = O.router(inp["x"], inp["w_router"], 3, gate, True)
    r1 = O.router(inp["x"], inp["w_router"], 3, gate, True, sel_bias=np.full(12, 0.375))
    np.testing.assert_array_equal(r0.topk_idx, r1.topk_idx)
    np.testing.assert_array_equal(r0.topk_w, r1.topk_w)


@pytest.mark.parametrize("gate", [O.GATE_SOFTMAX, O.GATE_SIGMOID])
def test_bias_moves_selection_only(gate):
    """Weights depend only on the chosen set and the unbiased scores.

    For each token, re-route it with a different bias that forces the same
    set (a large bonus on exactly the chosen experts).  The weights per expert
    must not change although the bias values differ completely.
    """
    rng = np.random.default_rng(3)
    E, k = 10, 3
    inp = _random_layer(rng, 60, 16, E, 4, k, bias=True)
    r = O.router(inp["x"], inp["w_router"], k, gate, True, inp["sel_bias"])
    changed = 0
    r_nobias = O.router(inp["x"], inp["w_router"], k, gate, True)
    for t in range(60):
        forced = np.zeros(E)
        forced[r.topk_idx[t]] = 1000.0
        rt = O.router(inp["x"][t:t + 1], inp["w_router"], k, gate, True, sel_bias=forced)
        assert set(rt.topk_idx[0]) == set(r.topk_idx[t])
        a = dict(zip(r.topk_idx[t].tolist(), r.topk_w[t].tolist()))
        b = dict(zip(rt.topk_idx[0].tolist(), rt.topk_w[0].tolist()))
        for e in a:
            assert abs(a[e] - b[e]) <= 1e-15
        changed += set(r.topk_idx[t]) != set(r_nobias.topk_idx[t])
    assert changed > 0, "the random bias should move at least one selection"


def test_topk_matches_full_python_sort():
    """Top-k = first k of a full sort by (-key, expert index); catches tie and order bugs."""
    rng = np.random.default_rng(4)
    E, k = 9, 4
    inp = _random_layer(rng, 200, 8, E, 4, k, bias=True)
    # plant exact ties between experts 2 and 5 and between 0 and 7
    inp["w_router"][5] = inp["w_router"][2]
    inp["sel_bias"][5] = inp["sel_bias"][2]
    inp["w_router"][7] = inp["w_router"][0]
    inp["sel_bias"][7] = inp["sel_bias"][0]
    r = O.router(inp["x"], inp["w_router"], k, O.GATE_SIGMOID, True, inp["sel_bias"])
    for t in range(200):
        keys = [math.fsum(float(a) * float(b) for a, b in zip(inp["x"][t], inp["w_router"][e]))
                + float(inp["sel_bias"][e]) for e in range(E)]
        ref = [e for _, e in sorted((-keys[e], e) for e in range(E))][:k]
        assert r.topk_idx[t].tolist() == ref


def test_logits_match_exactly_rounded_sums():
    """logits[t, e] = sum_c x[t,c] w[e,c]: compare with math.fsum (exact rounding)."""
    rng = np.random.default_rng(5)
    x = I.round_to_bf16(rng.standard_normal((7, 256)).astype(np.float32))
    w = I.round_to_bf16((0.02 * rng.standard_normal((5, 256))).astype(np.float32))
    r = O.router(x, w, 2, O.GATE_SOFTMAX, True)
    for t in range(7):
        for e in range(5):
            ref = math.fsum(float(a) * float(b) for a, b in zip(x[t], w[e]))
            assert abs(r.logits[t, e] - ref) <= 1e-13


def test_softmax_matches_scipy_and_is_shift_invariant():
    """Softmax over all experts (scipy reference); a constant logit offset changes nothing."""
    rng = np.random.default_rng(6)
    inp = _random_layer(rng, 100, 12, 8, 4, 8)
    r = O.router(inp["x"], inp["w_router"], 8, O.GATE_SOFTMAX, True)
    np.testing.assert_allclose(r.scores, scipy.special.softmax(r.logits, axis=1), rtol=1e-13)
    r2 = O.router(inp["x"], inp["w_router"], 8, O.GATE_SOFTMAX, True,
                  logit_offset=np.full(8, 3.25))
    np.testing.assert_allclose(r2.scores, r.scores, rtol=1e-13, atol=1e-16)
    np.testing.assert_array_equal(r2.topk_idx, r.topk_idx)
    # k = E with renormalisation: the weights are the full softmax row
    full = np.zeros_like(r.scores)
    np.put_along_axis(full, r.topk_idx, r.topk_w, axis=1)
    np.testing.assert_allclose(full, scipy.special.softmax(r.logits, axis=1), rtol=1e-8)


def test_sigmoid_matches_scipy_expit():
    rng = np.random.default_rng(7)
    inp = _random_layer(rng, 100, 12, 8, 4, 2)
    r = O.router(inp["x"], inp["w_router"], 2, O.GATE_SIGMOID, True)
    np.testing.assert_allclose(r.scores, scipy.special.expit(r.logits), rtol=1e-14)


def test_unnormalised_weights_are_raw_scores():
    rng = np.random.default_rng(8)
    inp = _random_layer(rng, 50, 12, 8, 4, 2)
    r = O.router(inp["x"], inp["w_router"], 2, O.GATE_SIGMOID, False)
    np.testing.assert_allclose(
        r.topk_w, scipy.special.expit(np.take_along_axis(r.logits, r.topk_idx, 1)), rtol=1e-14)


# --------------------------------------------------------------------------- #
# expert FFN                                                                  #
# --------------------------------------------------------------------------- #
def test_silu_closed_forms():
    z = np.array([0.0, math.log(3.0), -math.log(3.0), 40.0, -40.0])
    s = O.silu(z)
    assert s[0] == 0.0
    assert abs(s[1] - 0.75 * math.log(3.0)) < 1e-15
    assert abs(s[2] + 0.25 * math.log(3.0)) < 1e-15
    assert abs(s[3] - 40.0) < 1e-12 and abs(s[4]) < 1e-15
    zz = np.linspace(-8, 8, 33)
    # sigmoid(z) + sigmoid(-z) = 1, hence silu(z) - silu(-z) = z
    np.testing.assert_allclose(O.silu(zz) - O.silu(-zz), zz, atol=1e-14)


def test_swiglu_linear_in_up_not_in_gate():
    """Doubling w3 (up) doubles the output; doubling w1 (gate) does not: catches a gate/up swap."""
    rng = np.random.default_rng(9)
    x = rng.standard_normal((5, 6))
    w1, w3, w2 = rng.standard_normal((4, 6)), rng.standard_normal((4, 6)), rng.standard_normal((6, 4))
    y = O.swiglu_expert(x, w1, w3, w2)
    np.testing.assert_allclose(O.swiglu_expert(x, w1, 2 * w3, w2), 2 * y, rtol=1e-13)
    np.testing.assert_allclose(O.swiglu_expert(x, w1, w3, 3 * w2), 3 * y, rtol=1e-13)
    assert not np.allclose(O.swiglu_expert(x, 2 * w1, w3, w2), 2 * y, rtol=1e-3)


def test_swiglu_matches_torch_functional():
    """Same expert through torch's F.silu/F.linear in float64 (a library routine)."""
    import torch
    import torch.nn.functional as TF
    rng = np.random.default_rng(10)
    x = rng.standard_normal((9, 12))
    w1, w3, w2 = rng.standard_normal((7, 12)), rng.standard_normal((7, 12)), rng.standard_normal((12, 7))
    t = lambda a: torch.from_numpy(a)
    ref = TF.linear(TF.silu(TF.linear(t(x), t(w1))) * TF.linear(t(x), t(w3)), t(w2)).numpy()
    np.testing.assert_allclose(O.swiglu_expert(x, w1, w3, w2), ref, rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------- #
# layer                                                                       #
# --------------------------------------------------------------------------- #
@pytest.mark.parametrize("gate,shared,bias,offset,k",
                         [(O.GATE_SOFTMAX, False, False, False, 2),
                          (O.GATE_SIGMOID, True, True, False, 3),
                          (O.GATE_SIGMOID, True, True, True, 1),
                          (O.GATE_SOFTMAX, False, True, False, 6)])
def test_routed_equals_dense_masked_bruteforce(gate, shared, bias, offset, k):
    """Sorted-loop evaluation = every expert on every token, masked (tiny inputs)."""
    rng = np.random.default_rng(11 + k)
    inp = _random_layer(rng, 40, 16, 6, 8, k, shared, bias, offset)
    out, _ = O.moe_forward(inp, k, gate, True)
    ref = O.moe_forward_dense_masked(inp, k, gate, True)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)
    sub = [3, 17, 0, 39]
    part, _ = O.moe_forward(inp, k, gate, True, tokens=sub)
    np.testing.assert_allclose(part, ref[sub], rtol=1e-12, atol=1e-12)


def test_single_expert_top1_is_dense_swiglu():
    """E = 1, k = 1: the layer is one dense SwiGLU FFN scaled by 1/(1+1e-9)."""
    import torch
    import torch.nn.functional as TF
    rng = np.random.default_rng(12)
    inp = _random_layer(rng, 30, 10, 1, 6, 1)
    for gate in (O.GATE_SOFTMAX, O.GATE_SIGMOID):
        out, r = O.moe_forward(inp, 1, gate, True)
        t = lambda a: torch.from_numpy(np.ascontiguousarray(a))
        dense = TF.linear(TF.silu(TF.linear(t(inp["x"]), t(inp["w1"][0]))) *
                          TF.linear(t(inp["x"]), t(inp["w3"][0])), t(inp["w2"][0])).numpy()
        np.testing.assert_allclose(out, dense * r.topk_w, rtol=1e-12, atol=1e-12)
        assert np.all(np.abs(r.topk_w - 1.0) < 1e-8)


def test_expert_relabeling_invariance():
    """Permuting expert labels (router rows and weight stacks together) keeps the output."""
    rng = np.random.default_rng(13)
    inp = _random_layer(rng, 50, 12, 7, 5, 3, shared=True, bias=True)
    out, _ = O.moe_forward(inp, 3, O.GATE_SIGMOID, True)
    p = rng.permutation(7)
    inp2 = dict(inp)
    for key in ("w_router", "w1", "w3", "w2", "sel_bias"):
        inp2[key] = inp[key][p]
    out2, _ = O.moe_forward(inp2, 3, O.GATE_SIGMOID, True)
    np.testing.assert_allclose(out2, out, rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------- #
# dispatch                                                                    #
# --------------------------------------------------------------------------- #
def test_dispatch_matches_bucket_loop():
    """Stable (expert, token) order vs. per-expert buckets filled in token order."""
    rng = np.random.default_rng(14)
    T, E, k = 300, 11, 3
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)])
    dp = O.dispatch(idx, E)
    buckets = [[] for _ in range(E)]
    for t in range(T):
        for j in range(k):
            buckets[idx[t, j]].append((t, j))
    flat = [p for b in buckets for p in b]
    assert dp.counts.tolist() == [len(b) for b in buckets]
    assert dp.offsets[0] == 0 and dp.offsets[-1] == T * k
    assert dp.perm_src.tolist() == [t for t, _ in flat]
    assert dp.perm_expert.tolist() == [idx[t, j] for t, j in flat]
    for s, (t, j) in enumerate(flat):
        assert dp.slot_pos[t, j] == s
    assert sorted(dp.slot_pos.reshape(-1).tolist()) == list(range(T * k))


def test_combine_unpermutes_the_sorted_evaluation():
    """Routed outputs computed per expert in sorted row order, combined through
    slot_pos, equal the layer output; a one-hot k=1 combine is a row gather."""
    rng = np.random.default_rng(15)
    inp = _random_layer(rng, 40, 10, 5, 6, 2, shared=True, bias=True)
    out, r = O.moe_forward(inp, 2, O.GATE_SIGMOID, True)
    dp = O.dispatch(r.topk_idx, 5)
    y_perm = np.concatenate([
        O.swiglu_expert(inp["x"][dp.perm_src[dp.offsets[e]:dp.offsets[e + 1]]],
                        inp["w1"][e], inp["w3"][e], inp["w2"][e]) for e in range(5)])
    y_sh = O.swiglu_expert(inp["x"], inp["ws1"], inp["ws3"], inp["ws2"])
    np.testing.assert_allclose(O.combine(y_perm, dp.slot_pos, r.topk_w, y_sh), out,
                               rtol=1e-12, atol=1e-12)
    y = rng.standard_normal((7, 3))
    sp = np.array([[3], [0], [-1], [6]])
    g = O.combine(y, sp, np.ones((4, 1)))
    np.testing.assert_array_equal(g, np.stack([y[3], y[0], np.zeros(3), y[6]]))


def test_dispatch_rejects_bad_index():
    with pytest.raises(ValueError):
        O.dispatch(np.array([[0, 4]]), 4)


# --------------------------------------------------------------------------- #
# bias controller                                                             #
# --------------------------------------------------------------------------- #
def test_bias_uniform_counts_leave_bias_unchanged():
    b = np.array([0.25, -0.5, 1.0, 0.0], dtype=np.float32)
    out = O.bias_update(np.array([10, 10, 10, 10]), b)
    np.testing.assert_array_equal(out, b)


def test_bias_all_tokens_on_one_expert():
    """E=4, all load on expert 0: p = (1,0,0,0), err = (-0.75, 0.75, 0.75, 0.75)."""
    out = O.bias_update(np.array([40, 0, 0, 0]), np.zeros(4, np.float32), rate=1e-3)
    np.testing.assert_allclose(out, 1e-3 * np.array([-0.75, 0.75, 0.75, 0.75]), rtol=1e-6)
    assert out.dtype == np.float32


def test_bias_starved_boost_threshold():
    """Starved = load below 10% of the fair share gets +0.5 on its error."""
    E = 16
    c = np.array([100] * 14 + [0, 1])
    out = O.bias_update(c, np.zeros(E, np.float32), rate=1.0)
    # total 1401: loaded experts sit above the fair share 1/16, expert 14 has
    # no load, expert 15 has 1/1401 < 0.1/16 and is starved as well
    expect = [1 / 16 - 100 / 1401] * 14 + [1 / 16 + 0.5, 1 / 16 - 1 / 1401 + 0.5]
    np.testing.assert_allclose(out, expect, rtol=1e-6, atol=1e-7)
    assert out[14] > 0.5 and out[15] > 0.5 and out[0] < 0


def test_bias_empty_counts_and_clamp():
    """No tokens at all: total clamps to 1, every expert is starved; repeated steps saturate at +-10."""
    E = 8
    out = O.bias_update(np.zeros(E, np.int64), np.zeros(E, np.float32), rate=1.0)
    np.testing.assert_allclose(out, np.float32(1 / E + 0.5), rtol=1e-7)
    b = np.zeros(E, np.float32)
    for _ in range(40):
        b = O.bias_update(np.array([100, 0, 0, 0, 0, 0, 0, 0]), b, rate=1.0)
    assert b[0] == np.float32(-10.0) and np.all(b[1:] == np.float32(10.0))


# --------------------------------------------------------------------------- #
# page figures and load invariants                                            #
# --------------------------------------------------------------------------- #
def test_activated_width_invariant(figures):
    f = figures["activated_width"]
    w = I.WORKLOADS["wide"]
    assert (w.n_experts, w.d_ff, w.top_k) == (f["n_experts"], f["d_ff"], f["top_k"])
    assert w.top_k * w.d_ff == f["dense_width"]
    assert w.n_experts * w.d_ff == f["param_ratio"] * f["dense_width"]


def test_page2_workload_matches_config(figures):
    f = figures["page2_layer"]
    w = I.WORKLOADS["page2"]
    assert (w.d_model, w.n_experts, w.n_shared, w.top_k, w.d_ff) == (
        f["d_model"], f["n_experts"], f["n_shared"], f["top_k"], f["d_ff"])


def test_load_ceiling_on_skewed_workload(figures):
    """counts <= T, sum = T k, and max/(T k / E) <= E / k (= 10.67 at 64/6)."""
    f = figures["load_max_ratio_ceiling"]
    shp = I.WORKLOADS["skew"].replace(T=2048, d_model=256, d_ff=128, d_ff_shared=128)
    assert (shp.n_experts, shp.top_k) == (f["n_experts"], f["top_k"])
    inp = I.make_inputs(shp)
    r = O.router(inp["x"], inp["w_router"], shp.top_k, shp.gate, True,
                 inp.get("sel_bias"), inp.get("logit_offset"))
    c = O.dispatch(r.topk_idx, shp.n_experts).counts
    assert c.sum() == shp.T * shp.top_k and c.max() <= shp.T
    ratio = c.max() / (shp.T * shp.top_k / shp.n_experts)
    assert ratio <= f["ceiling"] + 0.005
    assert (c == 0).sum() > 0, "Zipf offsets should leave some experts without tokens"


def test_input_generator_is_bf16_exact_and_seeded():
    shp = I.WORKLOADS["page2"].replace(T=64)
    a = I.make_inputs(shp)
    b = I.make_inputs(shp)
    for key in a:
        np.testing.assert_array_equal(a[key], b[key])
    for key in ("x", "w_router", "w1", "w3", "w2", "ws1", "ws3", "ws2"):
        np.testing.assert_array_equal(I.round_to_bf16(a[key]), a[key])
    assert a["sel_bias"].min() >= -0.5 and a["sel_bias"].max() < 0.5


# --------------------------------------------------------------------------- #
# noaux_tc sign-style bias update (NEXT row: bias-rule variant)               #
# --------------------------------------------------------------------------- #
def test_sign_update_growth_matches_page_figure(figures):
    """64 micro-batch updates at rate 0.001 move a starved expert's bias by the
    page's 0.064 per optimizer step (and an overloaded one by -0.064)."""
    f = figures["noaux_tc_bias_growth"]
    counts = np.array([0, 500, 500, 1000])            # mean 500
    b = np.zeros(4, np.float32)
    for _ in range(f["accumulation_steps"]):
        b = O.bias_update_sign(counts, b, f["rate"])
    assert abs(b[0] - f["growth_per_optimizer_step"]) < 1e-6
    assert abs(b[3] + f["growth_per_optimizer_step"]) < 1e-6
    assert b[1] == 0.0 and b[2] == 0.0                # at the mean: no move


def test_sign_update_uniform_and_direction():
    b0 = np.array([0.5, -0.25, 0.0], np.float32)
    np.testing.assert_array_equal(O.bias_update_sign(np.array([7, 7, 7]), b0, 0.01), b0)
    out = O.bias_update_sign(np.array([1, 2, 9]), np.zeros(3, np.float32), 0.01)
    assert out[0] > 0 and out[1] > 0 and out[2] < 0
    np.testing.assert_allclose(np.abs(out), 0.01, rtol=1e-7)


# --------------------------------------------------------------------------- #
# router statistics (NEXT row)                                                #
# --------------------------------------------------------------------------- #
def _balanced_routing(T, E, k, logit=0.0, gate=O.GATE_SOFTMAX):
    """Token t picks experts (t*k + j) mod E: perfectly balanced counts."""
    x = np.zeros((T, 1))
    r = O.router(x, np.zeros((E, 1)), k, gate, True)
    r.logits[:] = logit
    r.scores[:] = (1.0 / E) if gate == O.GATE_SOFTMAX else 1.0 / (1.0 + math.exp(-logit))
    r.topk_idx[:] = (np.arange(T)[:, None] * k + np.arange(k)[None, :]) % E
    return r


def test_stats_closed_forms_balanced():
    T, E, k = 64, 8, 2
    st = O.router_stats(_balanced_routing(T, E, k))
    assert abs(st["z_loss"] - math.log(E) ** 2) < 1e-12      # lse of E zeros = ln E
    assert abs(st["aux_loss"] - k) < 1e-12                    # E * E * (k/E) * (1/E)
    assert st["cv"] == 0.0 and st["load_max_ratio"] == 1.0 and st["unused_frac"] == 0.0
    assert abs(st["entropy_bits"] - math.log2(E)) < 1e-12
    sg = O.router_stats(_balanced_routing(T, E, k, gate=O.GATE_SIGMOID))
    assert abs(sg["aux_loss"] - E * k / 2) < 1e-12            # sigmoid(0) = 1/2


def test_stats_collapse_hits_page_ceiling(figures):
    """Every token on the same k experts: load_max_ratio = E/k (64/6 = 10.67)."""
    f = figures["load_max_ratio_ceiling"]
    T, E, k = 30, f["n_experts"], f["top_k"]
    r = _balanced_routing(T, E, k)
    r.topk_idx[:] = np.arange(k)[None, :]
    st = O.router_stats(r)
    assert abs(st["load_max_ratio"] - E / k) < 1e-12 and abs(E / k - f["ceiling"]) < 0.005
    assert abs(st["unused_frac"] - (E - k) / E) < 1e-12


def test_stats_cv_uses_bessel_and_lse_matches_scipy():
    """cv of counts (1, 2, 3, 6): mean 3, unbiased std sqrt(14/3)."""
    r = _balanced_routing(12, 4, 1)
    r.topk_idx[:, 0] = np.array([0] + [1] * 2 + [2] * 3 + [3] * 6)
    assert abs(O.router_stats(r)["cv"] - math.sqrt(14 / 3) / 3) < 1e-12
    rng = np.random.default_rng(3)
    inp = _random_layer(rng, 50, 12, 7, 4, 2)
    rr = O.router(inp["x"], inp["w_router"], 2, O.GATE_SIGMOID, True)
    lse = scipy.special.logsumexp(rr.logits, axis=1)
    assert abs(O.router_stats(rr)["z_loss"] - np.mean(lse ** 2)) < 1e-12


# --------------------------------------------------------------------------- #
# selection-key variants: score-space bias, selection noise                  #
# --------------------------------------------------------------------------- #
@pytest.mark.parametrize("name", ["score_space_bias_sigmoid", "score_space_bias_softmax"])
def test_worked_score_space_bias(worked, name):
    """Catches: bias_space ignored, bias added to the weights, or the score
    transformation applied to the bias as well."""
    c = worked[name]
    x, w = _arr(c["x"]), _arr(c["w_router"])
    b = np.array(c["sel_bias"])
    for space, key in ((0, "logit_space"), (1, "score_space")):
        r = O.router(x, w, c["top_k"], _gate(c["gate"]), c["norm_topk_prob"], sel_bias=b,
                     bias_space=space)
        assert r.topk_idx.tolist() == c[key]["expected_idx"], key
        np.testing.assert_allclose(r.topk_w, _arr(c[key]["expected_w"]), rtol=0, atol=1e-15)


def test_worked_selection_noise(worked):
    """Catches: noise dropped, or noise leaking into the weights."""
    c = worked["selection_noise_moves_selection_only"]
    x, w = _arr(c["x"]), _arr(c["w_router"])
    r = O.router(x, w, c["top_k"], _gate(c["gate"]), c["norm_topk_prob"],
                 sel_noise=np.array(c["sel_noise"]))
    assert r.topk_idx.tolist() == c["expected_idx"]
    np.testing.assert_allclose(r.topk_w, _arr(c["expected_w"]), rtol=0, atol=1e-15)


@pytest.mark.parametrize("gate", [O.GATE_SOFTMAX, O.GATE_SIGMOID])
def test_score_space_without_bias_selects_like_logits(gate):
    """Both gates are increasing in each token's logits, so with no bias the
    score-space keys order the experts as the logits do.  Catches: a
    decreasing or mixed-up score transform in the keys."""
    rng = np.random.default_rng(7)
    x, w = rng.standard_normal((64, 16)), rng.standard_normal((24, 16))
    r0 = O.router(x, w, 5, gate, True)
    r1 = O.router(x, w, 5, gate, True, bias_space=1)
    np.testing.assert_array_equal(r0.topk_idx, r1.topk_idx)
    np.testing.assert_array_equal(r0.topk_w, r1.topk_w)


def test_token_constant_noise_equals_bias():
    """Noise that is the same for every token is a selection bias.  Catches:
    noise rows and columns transposed, or noise scaled twice."""
    rng = np.random.default_rng(8)
    x, w = rng.standard_normal((40, 12)), rng.standard_normal((10, 12))
    b = rng.uniform(-0.5, 0.5, 10)
    r_bias = O.router(x, w, 3, O.GATE_SIGMOID, True, sel_bias=b)
    r_noise = O.router(x, w, 3, O.GATE_SIGMOID, True, sel_noise=np.tile(b, (40, 1)))
    np.testing.assert_array_equal(r_bias.topk_idx, r_noise.topk_idx)
    np.testing.assert_array_equal(r_bias.topk_w, r_noise.topk_w)
    # and it moves nothing but the selection
    np.testing.assert_array_equal(r_noise.scores, O.router(x, w, 3, O.GATE_SIGMOID, True).scores)


# --------------------------------------------------------------------------- #
# layer backward                                                              #
# --------------------------------------------------------------------------- #
def _loss(inp, dout, top_k, gate, renorm, idx_fixed):
    out, r = O.moe_forward(inp, top_k, gate, renorm)
    assert np.array_equal(r.topk_idx, idx_fixed), "perturbation changed the selection"
    return float(np.sum(dout * out))


@pytest.mark.parametrize("gate,renorm,shared", [(O.GATE_SIGMOID, True, True),
                                                (O.GATE_SOFTMAX, True, False),
                                                (O.GATE_SOFTMAX, False, True),
                                                (O.GATE_SIGMOID, False, False)])
def test_backward_matches_central_differences(gate, renorm, shared):
    """Every gradient the oracle returns equals the central difference of
    <dout, out> computed from the forward alone.  Catches: a dropped term of
    the SwiGLU chain rule, the renormalisation Jacobian, a transposed weight
    gradient, or a missing router / shared-expert contribution to dx."""
    rng = np.random.default_rng(11 + gate + 2 * renorm)
    T, d, E, F, k = 6, 5, 4, 3, 2
    inp = _random_layer(rng, T, d, E, F, k, shared=shared, bias=True, offset=True)
    dout = rng.standard_normal((T, d))
    r = O.router(inp["x"], inp["w_router"], k, gate, renorm, inp["sel_bias"],
                 inp["logit_offset"])
    assert np.all(r.edge_gap > 1e-3)     # no selection change under the perturbation
    g = O.moe_backward(inp, k, gate, renorm, dout)
    names = ["x", "w_router", "w1", "w3", "w2"] + (["ws1", "ws3", "ws2"] if shared else [])
    grad_key = {"x": "dx", "w_router": "dw_router", "w1": "dw1", "w3": "dw3", "w2": "dw2",
                "ws1": "dws1", "ws3": "dws3", "ws2": "dws2"}
    h = 1e-6
    for name in names:
        base = inp[name]
        num = np.zeros(base.shape)
        for pos in np.ndindex(base.shape):
            p = dict(inp)
            a = base.copy(); a[pos] += h; p[name] = a
            lp = _loss(p, dout, k, gate, renorm, r.topk_idx)
            a = base.copy(); a[pos] -= h; p[name] = a
            lm = _loss(p, dout, k, gate, renorm, r.topk_idx)
            num[pos] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(g[grad_key[name]], num, rtol=1e-6, atol=1e-7, err_msg=name)


def test_backward_bias_and_offset_get_no_gradient_through_selection():
    """The bias only moves the selection: with the selection unchanged, the
    loss does not depend on it at all (zero central difference).  Catches: the
    bias leaking into the weights and hence into the gradients."""
    rng = np.random.default_rng(5)
    inp = _random_layer(rng, 6, 5, 4, 3, 2, bias=True)
    dout = rng.standard_normal((6, 5))
    r = O.router(inp["x"], inp["w_router"], 2, O.GATE_SIGMOID, True, inp["sel_bias"])
    assert np.all(r.edge_gap > 1e-3)
    l0 = _loss(inp, dout, 2, O.GATE_SIGMOID, True, r.topk_idx)
    for e in range(4):
        p = dict(inp)
        b = inp["sel_bias"].copy(); b[e] += 1e-7; p["sel_bias"] = b
        assert _loss(p, dout, 2, O.GATE_SIGMOID, True, r.topk_idx) == l0


def test_backward_top1_renormalised_has_no_router_gradient():
    """With top-1 and renormalisation every weight is s / (s + 1e-9), almost
    exactly 1, so the router gradient is (almost exactly) zero.  Catches a
    renormalisation Jacobian with the wrong sign or a missing term."""
    rng = np.random.default_rng(9)
    inp = _random_layer(rng, 8, 6, 5, 4, 1)
    dout = rng.standard_normal((8, 6))
    g = O.moe_backward(inp, 1, O.GATE_SOFTMAX, True, dout)
    assert np.max(np.abs(g["dw_router"])) < 1e-7


def test_near_tie_table_is_the_oracles():
    """tests/golden/near_ties.json (written by make_near_ties.py from the
    oracle alone): its rule, its workloads, and the tiny workload's entry
    recomputed here (the full-size entries are recomputed by the GPU parity
    tests, which route those workloads with the oracle anyway)."""
    import json
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "near_ties.json")
    with open(path) as f:
        table = json.load(f)
    assert "1e-6" in table["rule"]
    assert set(table["workloads"]) == set(I.WORKLOAD_ORDER)
    for name, e in table["workloads"].items():
        assert e["T"] == I.WORKLOADS[name].T and e["excluded"] == len(e["tokens"])
    shape = I.WORKLOADS["tiny"]
    host = I.make_inputs(shape)
    r = O.router(host["x"], host["w_router"], shape.top_k, shape.gate, True)
    assert (r.edge_gap < 1e-6).nonzero()[0].tolist() == table["workloads"]["tiny"]["tokens"]
