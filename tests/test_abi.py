"""C ABI checks that need no GPU: the library loads, exports every function the
header declares, and rejects bad arguments before launching anything."""
import ctypes

import pytest

from mixture_experts_ffn_bias_b200 import binding as B
from mixture_experts_ffn_bias_b200 import build as build_mod
from mixture_experts_ffn_bias_b200 import inputs as I


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return B.lib()


def test_header_symbols_exported(lib):
    names = B.header_functions()
    assert {"moe_router_topk", "moe_permute", "moe_grouped_swiglu", "moe_combine",
            "moe_bias_update", "moe_forward", "moe_workspace_size", "moe_device_status",
            "moe_status_string", "moe_check_config"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_struct_layout():
    assert ctypes.sizeof(B.MoEConfig) == 40
    assert ctypes.sizeof(B.MoEExpertWeights) == 6 * ctypes.sizeof(ctypes.c_void_p)
    assert ctypes.sizeof(B.MoEExpertGrads) == 6 * ctypes.sizeof(ctypes.c_void_p)
    # moe_router_opts: int32 bias_space, int32 reserved, const float* sel_noise
    assert ctypes.sizeof(B.MoERouterOpts) == 8 + ctypes.sizeof(ctypes.c_void_p)
    assert B.MoERouterOpts.sel_noise.offset == 8


@pytest.mark.parametrize("name", I.WORKLOAD_ORDER)
def test_workloads_are_accepted(lib, name):
    cfg = B.config_from_shape(I.WORKLOADS[name])
    assert B.moe_check_config(cfg) == B.MOE_OK
    assert B.moe_workspace_size(cfg) > 0


def test_workspace_size_grows_with_tokens(lib):
    shp = I.WORKLOADS["qwen3_30b"]
    a = B.moe_workspace_size(B.config_from_shape(shp, T=1024))
    b = B.moe_workspace_size(B.config_from_shape(shp, T=2048))
    assert b > a
    # x_perm and y_perm alone are 2 * T*k*d bf16
    assert b >= 2 * 2048 * 8 * 2048 * 2


@pytest.mark.parametrize("field,value,expect", [
    ("top_k", 0, B.MOE_ERR_INVALID),
    ("top_k", 17, B.MOE_ERR_INVALID),          # k > E
    ("n_experts", 0, B.MOE_ERR_INVALID),
    ("T", -1, B.MOE_ERR_INVALID),
    ("gate", 7, B.MOE_ERR_INVALID),
    ("dtype", 3, B.MOE_ERR_INVALID),
    ("n_shared", 2, B.MOE_ERR_INVALID),
    ("d_model", 100, B.MOE_ERR_UNSUPPORTED),   # bf16 rows must be multiples of 128
    ("d_ff", 1000, B.MOE_ERR_UNSUPPORTED),
])
def test_config_validation(lib, field, value, expect):
    cfg = B.config_from_shape(I.WORKLOADS["page2"])
    setattr(cfg, field, value)
    assert B.moe_check_config(cfg) == expect
    assert B.moe_workspace_size(cfg) == 0


def test_too_many_experts_unsupported(lib):
    cfg = B.make_config(64, 128, 300, 128, 2)
    assert B.moe_check_config(cfg) == B.MOE_ERR_UNSUPPORTED


class _FakeTensor:
    """Host-side stand-in carrying an address only; never dereferenced because
    every case below fails validation before any CUDA call."""

    def __init__(self, addr, nbytes=0):
        self._a, self._n = addr, nbytes

    def data_ptr(self):
        return self._a

    def numel(self):
        return self._n

    def element_size(self):
        return 1


def test_null_and_misaligned_pointers_rejected(lib):
    cfg = B.config_from_shape(I.WORKLOADS["page2"])
    ok = _FakeTensor(1 << 20)
    ws = _FakeTensor(1 << 20, B.moe_workspace_size(cfg))
    st = B.moe_router_topk(cfg, None, ok, None, None, ok, ok, ws, stream=0, check=False)
    assert st == B.MOE_ERR_INVALID
    st = B.moe_router_topk(cfg, _FakeTensor((1 << 20) + 8), ok, None, None, ok, ok, ws,
                           stream=0, check=False)
    assert st == B.MOE_ERR_INVALID
    # workspace too small
    st = B.moe_router_topk(cfg, ok, ok, None, None, ok, ok, _FakeTensor(1 << 20, 1024),
                           stream=0, check=False)
    assert st == B.MOE_ERR_WORKSPACE
    # key-variant router: bias_space outside {0, 1}, misaligned noise
    st = B.moe_router_topk_opts(cfg, ok, ok, None, None, ok, ok, ws, bias_space=2, stream=0,
                                check=False)
    assert st == B.MOE_ERR_INVALID
    st = B.moe_router_topk_opts(cfg, ok, ok, None, None, ok, ok, ws, bias_space=1,
                                sel_noise=_FakeTensor((1 << 20) + 2), stream=0, check=False)
    assert st == B.MOE_ERR_INVALID
    st = B.moe_router_topk_opts(cfg, None, ok, None, None, ok, ok, ws, bias_space=1, stream=0,
                                check=False)
    assert st == B.MOE_ERR_INVALID
    # shared expert weights missing for a layer with a shared expert
    w = {"w1": ok, "w3": ok, "w2": ok}
    st = B.moe_forward(cfg, ok, ok, None, None, w, ok, ok, ok, ok, ws, stream=0, check=False)
    assert st == B.MOE_ERR_INVALID
    # y_shared given although the layer has no shared expert
    cfg3 = B.config_from_shape(I.WORKLOADS["qwen3_30b"])
    st = B.moe_combine(cfg3, ok, ok, ok, ok, ok, stream=0, check=False)
    assert st == B.MOE_ERR_INVALID
    with pytest.raises(B.MoEError):
        B.moe_combine(cfg3, ok, ok, ok, ok, ok, stream=0)


def test_status_strings(lib):
    for s in range(7):
        assert B.status_string(s) and B.status_string(s) != "unknown status"
    assert B.status_string(99) == "unknown status"


def test_backward_arguments_validated(lib):
    shape = I.WORKLOADS["page2"]
    cfg = B.config_from_shape(shape)
    ok = _FakeTensor(1 << 20, 1 << 40)
    w = {"w1": ok, "w3": ok, "w2": ok, "ws1": ok, "ws3": ok, "ws2": ok}
    g = {"dw1": ok, "dw3": ok, "dw2": ok, "dws1": ok, "dws3": ok, "dws2": ok}
    # shared-expert gradients missing for a layer with a shared expert
    g2 = {"dw1": ok, "dw3": ok, "dw2": ok}
    st = B.moe_backward(cfg, ok, ok, None, w, ok, ok, ok, ok, ok, g2, ok, ok, stream=0,
                        check=False)
    assert st == B.MOE_ERR_INVALID
    # backward scratch too small
    st = B.moe_backward(cfg, ok, ok, None, w, ok, ok, ok, ok, ok, g, ok, _FakeTensor(1 << 20, 256),
                        stream=0, check=False)
    assert st == B.MOE_ERR_WORKSPACE
    # fp32 layers have no backward
    cfg32 = B.config_from_shape(I.WORKLOADS["tiny"])
    assert B.moe_backward_workspace_size(cfg32) == 0
    st = B.moe_backward(cfg32, ok, ok, None, w, ok, ok, ok, ok, ok, g, ok, ok, stream=0,
                        check=False)
    assert st == B.MOE_ERR_UNSUPPORTED


def test_forward_options_layout_and_validation(lib):
    assert ctypes.sizeof(B.MoEForwardOpts) == 16
    cfg = B.config_from_shape(I.WORKLOADS["page2"])
    ok = _FakeTensor(1 << 20)
    ws = _FakeTensor(1 << 20, B.moe_workspace_size(cfg))
    w = {k: ok for k in ("w1", "w3", "w2", "ws1", "ws3", "ws2")}
    st = B.moe_forward_ex(cfg, ok, ok, None, None, w, ok, ok, ok, ok, ws, gather_rows=2,
                          stream=0, check=False)
    assert st == B.MOE_ERR_INVALID
    tiny = B.config_from_shape(I.WORKLOADS["tiny"])
    ws32 = _FakeTensor(1 << 20, B.moe_workspace_size(tiny))
    st = B.moe_forward_ex(tiny, ok, ok, None, None, w, ok, ok, ok, ok, ws32, gather_rows=1,
                          stream=0, check=False)
    assert st == B.MOE_ERR_UNSUPPORTED
    st = B.moe_forward_ex(cfg, ok, ok, None, None, w, ok, ok, ok, ok, ws, fold_combine=2,
                          stream=0, check=False)
    assert st == B.MOE_ERR_INVALID
    st = B.moe_forward_ex(tiny, ok, ok, None, None, w, ok, ok, ok, ok, ws32, fold_combine=1,
                          stream=0, check=False)
    assert st == B.MOE_ERR_UNSUPPORTED
    st = B.moe_forward_ex(cfg, ok, ok, None, None, w, ok, ok, ok, ok, ws, scatter_in_gemm=2,
                          stream=0, check=False)
    assert st == B.MOE_ERR_INVALID
    st = B.moe_forward_ex(cfg, ok, ok, None, None, w, ok, ok, ok, ok, ws, gather_rows=1,
                          scatter_in_gemm=1, stream=0, check=False)
    assert st == B.MOE_ERR_INVALID
    st = B.moe_forward_ex(tiny, ok, ok, None, None, w, ok, ok, ok, ok, ws32, scatter_in_gemm=1,
                          stream=0, check=False)
    assert st == B.MOE_ERR_UNSUPPORTED
    opts = B.MoEForwardOpts(0, 0, 0)
    opts.reserved[0] = 1
    st = B.lib().moe_forward_ex(ctypes.byref(cfg), None, None, None, None,
                                ctypes.byref(B.expert_weights(w)), None, None, None, None,
                                ctypes.byref(opts), None, 0, None)
    assert st == B.MOE_ERR_INVALID


def test_forward_dispatch_view_points_into_the_workspace(lib):
    """Host arithmetic only: the three regions lie inside ws, in order, are
    256-byte aligned and large enough for offsets [E+1], slot_pos [T, k] and
    perm_src [T*k]."""
    shape = I.WORKLOADS["qwen3_30b"]
    cfg = B.config_from_shape(shape)
    n = B.moe_workspace_size(cfg)
    base = 1 << 30
    ptrs = [ctypes.c_void_p(0) for _ in range(3)]
    st = lib.moe_forward_dispatch_view(ctypes.byref(cfg), base, n, *[ctypes.byref(p) for p in ptrs])
    assert st == B.MOE_OK
    offs, slot, src = (p.value - base for p in ptrs)
    E, R = shape.n_experts, shape.T * shape.top_k
    assert 0 < offs and offs + 4 * (E + 1) <= slot and slot + 4 * R <= src
    assert src + 4 * R <= n
    assert offs % 256 == slot % 256 == src % 256 == 0
    assert lib.moe_forward_dispatch_view(ctypes.byref(cfg), base, n - 1,
                                         *[ctypes.byref(p) for p in ptrs]) == B.MOE_ERR_WORKSPACE
    assert lib.moe_forward_dispatch_view(ctypes.byref(cfg), base + 8, n,
                                         *[ctypes.byref(p) for p in ptrs]) == B.MOE_ERR_INVALID
