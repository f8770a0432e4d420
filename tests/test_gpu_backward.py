"""Backward of the layer (moe_backward, through the C ABI) against the fp64
oracle's gradients (oracle.moe_backward, pinned by central differences):
dx, the router weight gradient and every expert weight gradient, element by
element over the whole tensors, on small shapes that span several tiles with
ragged expert segments and on the full benchmark workload."""
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

# activation gradients pass through five bf16 roundings (dY, dH, G/U, dG/dU,
# dX) and the weight gradients are stored in bf16
GRAD_TOL = 3e-2

SMALL = {
    "page2_small": I.WORKLOADS["page2"].replace(T=640),
    "qwen3_small": I.WORKLOADS["qwen3_30b"].replace(T=600, d_model=256, d_ff=256),
    "wide_small": I.WORKLOADS["wide"].replace(T=200, d_model=512, d_ff=384),
    "skew_small": I.WORKLOADS["skew"].replace(T=1000, d_model=256, d_ff=256, d_ff_shared=256),
}


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build_mod.build()
    B.lib()


def _np(t):
    return t.detach().float().cpu().numpy()


@pytest.mark.parametrize("name,mode", [(n, "default") for n in SMALL] +
                         [("qwen3_small", "gather"), ("skew_small", "gather"),
                          ("qwen3_small", "scatter_in_gemm"), ("page2_small", "scatter_in_gemm")])
def test_backward_small_elementwise(name, mode):
    """mode gather: the forward ran with gathered gate/up rows (no permuted
    copy of x kept), and the backward gathers x's rows itself;
    scatter_in_gemm: the forward's gate/up GEMM filled the permuted copy the
    backward reads."""
    shape = SMALL[name]
    host = I.make_inputs(shape)
    layer = MoELayer(shape, host)
    layer.forward(gather_rows=mode == "gather", scatter_in_gemm=mode == "scatter_in_gemm")
    dout_h = I.round_to_bf16(np.random.default_rng(77).standard_normal(
        (shape.T, shape.d_model)).astype(np.float32))
    g = layer.backward(to_device(dout_h, torch.bfloat16, "cuda"))
    torch.cuda.synchronize()
    st, flags = B.moe_device_status(layer.bws)
    assert st == B.MOE_OK, (st, flags)
    r = P.oracle_routing(shape, host)
    np.testing.assert_array_equal(_np(layer.topk_idx), r.topk_idx)   # no near ties here
    ref = O.moe_backward(host, shape.top_k, shape.gate, bool(shape.norm_topk_prob), dout_h,
                         routing=r)
    checks = [("dx", "dx"), ("dw_router", "dw_router"), ("dw1", "dw1"), ("dw3", "dw3"),
              ("dw2", "dw2")]
    if shape.n_shared:
        checks += [("dws1", "dws1"), ("dws3", "dws3"), ("dws2", "dws2")]
    for gk, rk in checks:
        err = P.rel_err(_np(g[gk]), ref[rk])
        assert err <= GRAD_TOL, f"{gk}: relative error {err:.3e}"


@pytest.mark.parametrize("name", ["page2", "qwen3_30b", "skew", "wide"])
def test_backward_full_size_every_element(name):
    """Full-size workloads (qwen3_30b is the one the benchmark's backward
    mode times, in the same configuration): every element of dx, the router
    weight gradient and every expert weight gradient (the shared expert's
    too, on page2 and skew) against the oracle.  The stored near-tie lists of these
    workloads are empty, so the GPU's routing is the oracle's on every token
    (checked)."""
    shape = I.WORKLOADS[name]
    host = I.make_inputs(shape)
    layer = MoELayer(shape, host)
    layer.forward()
    dout_h = I.round_to_bf16(np.random.default_rng(78).standard_normal(
        (shape.T, shape.d_model)).astype(np.float32))
    g = layer.backward(to_device(dout_h, torch.bfloat16, "cuda"))
    torch.cuda.synchronize()
    st, flags = B.moe_device_status(layer.bws)
    assert st == B.MOE_OK, (st, flags)
    r = P.oracle_routing(shape, host)
    np.testing.assert_array_equal(_np(layer.topk_idx), r.topk_idx)
    keys = ["dx", "dw_router", "dw1", "dw3", "dw2"]
    if shape.n_shared:
        keys += ["dws1", "dws3", "dws2"]
    got = {k: _np(g[k]) for k in keys}
    del layer, g
    torch.cuda.empty_cache()
    ref = O.moe_backward(host, shape.top_k, shape.gate, bool(shape.norm_topk_prob), dout_h,
                         routing=r)
    for k, v in got.items():
        err = P.rel_err(v, ref[k])
        print(f"{name} backward {k}: relative error {err:.3e}")
        assert err <= GRAD_TOL, f"{k}: relative error {err:.3e}"


def test_backward_rejects_fp32_layer():
    shape = I.WORKLOADS["tiny"]
    assert B.moe_backward_workspace_size(B.config_from_shape(shape)) == 0
