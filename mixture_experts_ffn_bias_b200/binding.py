"""Python binding of libmoe_b200.so (the C ABI declared in include/moe.h).

Argument marshalling only: every function takes torch CUDA tensors (or None
for optional pointers), passes their device addresses and sizes to the C entry
point of the same name, and raises :class:`MoEError` on a non-zero status
unless ``check=False``.  All arithmetic happens in the library's CUDA kernels;
there is no fallback.  ``stream=None`` means torch's current stream.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Dict, Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoe_b200.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "moe.h")

MOE_OK = 0
MOE_ERR_INVALID = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_WORKSPACE = 3
MOE_ERR_CUDA = 4
MOE_ERR_TIMEOUT = 5
MOE_ERR_DATA = 6

GATE_SOFTMAX = 0
GATE_SIGMOID = 1
NOALLOC_MAX_BLOCK_COUNTS = 262144   # MOE_PERMUTE_NOALLOC_MAX_BLOCK_COUNTS in moe.h
DTYPE_F32 = 0
DTYPE_BF16 = 1


class MoEError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{msg} (status {status})")
        self.status = status


class MoEConfig(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "T", "d_model", "n_experts", "d_ff", "top_k", "n_shared", "d_ff_shared",
        "gate", "norm_topk_prob", "dtype")]


class MoEExpertWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("w1", "w3", "w2", "ws1", "ws3", "ws2")]


class MoEExpertGrads(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("dw1", "dw3", "dw2", "dws1", "dws3", "dws2")]


class MoEForwardOpts(ctypes.Structure):
    _fields_ = [("gather_rows", ctypes.c_int32), ("fold_combine", ctypes.c_int32),
                ("scatter_in_gemm", ctypes.c_int32), ("reserved", ctypes.c_int32 * 1)]


class MoERouterOpts(ctypes.Structure):
    _fields_ = [("bias_space", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("sel_noise", ctypes.c_void_p)]


_VP, _SZ, _I32, _F64 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_double
_CFG = ctypes.POINTER(MoEConfig)
_WTS = ctypes.POINTER(MoEExpertWeights)
_SIGNATURES = {
    "moe_workspace_size": (_SZ, [_CFG]),
    "moe_check_config": (_I32, [_CFG]),
    "moe_router_topk": (_I32, [_CFG, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "moe_router_topk_opts": (_I32, [_CFG, _VP, _VP, _VP, _VP, ctypes.POINTER(MoERouterOpts),
                                     _VP, _VP, _VP, _SZ, _VP]),
    "moe_router_logits": (_I32, [_CFG, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "moe_router_stats": (_I32, [_CFG, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "moe_permute": (_I32, [_CFG, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "moe_grouped_swiglu": (_I32, [_CFG, _VP, _VP, _WTS, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "moe_combine": (_I32, [_CFG, _VP, _VP, _VP, _VP, _VP, _VP]),
    "moe_bias_update": (_I32, [_CFG, _VP, _VP, _F64, _F64, _F64, _F64, _VP]),
    "moe_bias_update_sign": (_I32, [_CFG, _VP, _VP, _F64, _VP]),
    "moe_forward": (_I32, [_CFG, _VP, _VP, _VP, _VP, _WTS, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "moe_forward_profiled": (_I32, [_CFG, _VP, _VP, _VP, _VP, _WTS, _VP, _VP, _VP, _VP, _VP, _SZ,
                                     _VP, ctypes.POINTER(ctypes.c_void_p)]),
    "moe_forward_ex": (_I32, [_CFG, _VP, _VP, _VP, _VP, _WTS, _VP, _VP, _VP, _VP,
                               ctypes.POINTER(MoEForwardOpts), _VP, _SZ, _VP]),
    "moe_forward_dispatch_view": (_I32, [_CFG, _VP, _SZ, ctypes.POINTER(_VP),
                                          ctypes.POINTER(_VP), ctypes.POINTER(_VP)]),
    "moe_permute_noalloc": (_I32, [_CFG, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP]),
    "moe_device_status": (_I32, [_VP, _SZ, _VP, ctypes.POINTER(ctypes.c_uint32)]),
    "moe_router_refined_tokens": (_I32, [_VP, _SZ, _VP, ctypes.POINTER(ctypes.c_int32)]),
    "moe_selftest_bounded_wait": (_I32, [_VP, _SZ, _F64, _VP]),
    "moe_status_string": (ctypes.c_char_p, [_I32]),
    "moe_backward_workspace_size": (_SZ, [_CFG]),
    "moe_backward": (_I32, [_CFG, _VP, _VP, _VP, _WTS, _VP, _VP, _VP, _VP, _VP,
                            ctypes.POINTER(MoEExpertGrads), _VP, _SZ, _VP, _SZ, _VP]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """Load the library (it must have been built; there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m mixture_experts_ffn_bias_b200.build` (needs nvcc)")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def header_functions() -> list:
    """Names of the functions include/moe.h declares."""
    with open(HEADER) as f:
        text = f.read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w\*]+\s+\**(moe_\w+)\s*\(", text, re.M)))


def status_string(st: int) -> str:
    return lib().moe_status_string(int(st)).decode()


def _check(st: int, check: bool) -> int:
    if check and st != MOE_OK:
        raise MoEError(st, status_string(st))
    return st


def make_config(T, d_model, n_experts, d_ff, top_k, n_shared=0, d_ff_shared=0,
                gate=GATE_SOFTMAX, norm_topk_prob=1, dtype=DTYPE_BF16) -> MoEConfig:
    return MoEConfig(T, d_model, n_experts, d_ff, top_k, n_shared,
                     d_ff_shared if n_shared else 0, gate, norm_topk_prob, dtype)


def config_from_shape(shape, T: Optional[int] = None) -> MoEConfig:
    """MoEConfig for a workload of mixture_experts_ffn_bias_b200.inputs."""
    return make_config(shape.T if T is None else T, shape.d_model, shape.n_experts,
                       shape.d_ff, shape.top_k, shape.n_shared, shape.d_ff_shared,
                       shape.gate, shape.norm_topk_prob, shape.dtype)


def _p(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _s(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def _nbytes(ws) -> int:
    return ws.numel() * ws.element_size()


def expert_weights(w: Dict) -> MoEExpertWeights:
    return MoEExpertWeights(_p(w["w1"]), _p(w["w3"]), _p(w["w2"]),
                            _p(w.get("ws1")), _p(w.get("ws3")), _p(w.get("ws2")))


def moe_workspace_size(cfg: MoEConfig) -> int:
    return int(lib().moe_workspace_size(ctypes.byref(cfg)))


def moe_check_config(cfg: MoEConfig) -> int:
    return int(lib().moe_check_config(ctypes.byref(cfg)))


def moe_router_topk(cfg, x, w_router, sel_bias, logit_offset, topk_idx, topk_w, ws,
                    stream=None, check=True) -> int:
    st = lib().moe_router_topk(ctypes.byref(cfg), _p(x), _p(w_router), _p(sel_bias),
                               _p(logit_offset), _p(topk_idx), _p(topk_w), _p(ws),
                               _nbytes(ws) if ws is not None else 0, _s(stream))
    return _check(st, check)


def moe_router_topk_opts(cfg, x, w_router, sel_bias, logit_offset, topk_idx, topk_w, ws,
                         bias_space=0, sel_noise=None, stream=None, check=True) -> int:
    """moe_router_topk with the key variants: bias_space 1 puts the bias on
    the gate scores; sel_noise ([T, E] fp32, already scaled) is added to the
    keys."""
    opts = MoERouterOpts(int(bias_space), 0, _p(sel_noise))
    st = lib().moe_router_topk_opts(ctypes.byref(cfg), _p(x), _p(w_router), _p(sel_bias),
                                    _p(logit_offset), ctypes.byref(opts), _p(topk_idx),
                                    _p(topk_w), _p(ws), _nbytes(ws) if ws is not None else 0,
                                    _s(stream))
    return _check(st, check)


def moe_router_logits(cfg, x, w_router, logit_offset, logits, ws, stream=None, check=True) -> int:
    st = lib().moe_router_logits(ctypes.byref(cfg), _p(x), _p(w_router), _p(logit_offset),
                                 _p(logits), _p(ws), _nbytes(ws) if ws is not None else 0,
                                 _s(stream))
    return _check(st, check)


def moe_router_stats(cfg, x, w_router, logit_offset, topk_idx, stats, ws, stream=None,
                     check=True) -> int:
    st = lib().moe_router_stats(ctypes.byref(cfg), _p(x), _p(w_router), _p(logit_offset),
                                _p(topk_idx), _p(stats), _p(ws),
                                _nbytes(ws) if ws is not None else 0, _s(stream))
    return _check(st, check)


STAT_NAMES = ("z_loss", "aux_loss", "cv", "entropy_bits", "load_max_ratio", "unused_frac")


def moe_permute(cfg, topk_idx, x, counts, offsets, slot_pos, perm_src, x_perm, ws,
                stream=None, check=True) -> int:
    st = lib().moe_permute(ctypes.byref(cfg), _p(topk_idx), _p(x), _p(counts), _p(offsets),
                           _p(slot_pos), _p(perm_src), _p(x_perm), _p(ws),
                           _nbytes(ws) if ws is not None else 0, _s(stream))
    return _check(st, check)


def moe_permute_noalloc(cfg, topk_idx, x, counts, offsets, slot_pos, perm_src, x_perm,
                        stream=None, check=True) -> int:
    """moe_permute with its scratch in the library's fixed device array (no workspace)."""
    st = lib().moe_permute_noalloc(ctypes.byref(cfg), _p(topk_idx), _p(x), _p(counts),
                                   _p(offsets), _p(slot_pos), _p(perm_src), _p(x_perm),
                                   _s(stream))
    return _check(st, check)


def moe_grouped_swiglu(cfg, x_perm, offsets, weights: Dict, x, y_perm, y_shared, ws,
                       stream=None, check=True) -> int:
    w = expert_weights(weights)
    st = lib().moe_grouped_swiglu(ctypes.byref(cfg), _p(x_perm), _p(offsets), ctypes.byref(w),
                                  _p(x), _p(y_perm), _p(y_shared), _p(ws),
                                  _nbytes(ws) if ws is not None else 0, _s(stream))
    return _check(st, check)


def moe_combine(cfg, y_perm, slot_pos, topk_w, y_shared, out, stream=None, check=True) -> int:
    st = lib().moe_combine(ctypes.byref(cfg), _p(y_perm), _p(slot_pos), _p(topk_w),
                           _p(y_shared), _p(out), _s(stream))
    return _check(st, check)


def moe_bias_update(cfg, counts, sel_bias, rate=1e-3, starved_frac=0.1, starved_add=0.5,
                    clamp=10.0, stream=None, check=True) -> int:
    st = lib().moe_bias_update(ctypes.byref(cfg), _p(counts), _p(sel_bias), rate,
                               starved_frac, starved_add, clamp, _s(stream))
    return _check(st, check)


def moe_bias_update_sign(cfg, counts, sel_bias, rate=1e-3, stream=None, check=True) -> int:
    st = lib().moe_bias_update_sign(ctypes.byref(cfg), _p(counts), _p(sel_bias), rate, _s(stream))
    return _check(st, check)


def moe_forward(cfg, x, w_router, sel_bias, logit_offset, weights: Dict, out, topk_idx,
                topk_w, counts, ws, stream=None, check=True) -> int:
    w = expert_weights(weights)
    st = lib().moe_forward(ctypes.byref(cfg), _p(x), _p(w_router), _p(sel_bias),
                           _p(logit_offset), ctypes.byref(w), _p(out), _p(topk_idx),
                           _p(topk_w), _p(counts), _p(ws),
                           _nbytes(ws) if ws is not None else 0, _s(stream))
    return _check(st, check)


def moe_forward_ex(cfg, x, w_router, sel_bias, logit_offset, weights: Dict, out, topk_idx,
                   topk_w, counts, ws, gather_rows=0, fold_combine=0, scatter_in_gemm=0,
                   stream=None, check=True) -> int:
    """moe_forward with the expert-path options (gather_rows=1: the gate/up
    GEMM gathers its rows from x instead of reading a permuted copy;
    fold_combine=1: the down GEMM forms the combined output itself;
    scatter_in_gemm=1: the gate/up GEMM fills the permuted copy while it
    runs)."""
    w = expert_weights(weights)
    opts = MoEForwardOpts(int(gather_rows), int(fold_combine), int(scatter_in_gemm))
    st = lib().moe_forward_ex(ctypes.byref(cfg), _p(x), _p(w_router), _p(sel_bias),
                              _p(logit_offset), ctypes.byref(w), _p(out), _p(topk_idx),
                              _p(topk_w), _p(counts), ctypes.byref(opts), _p(ws),
                              _nbytes(ws) if ws is not None else 0, _s(stream))
    return _check(st, check)


def moe_forward_dispatch_view(cfg, ws):
    """(offsets, slot_pos, perm_src) int32 views into the forward's workspace
    ``ws`` (a torch uint8 tensor): the routed order the last forward wrote."""
    import torch
    ptrs = [ctypes.c_void_p(0) for _ in range(3)]
    _check(lib().moe_forward_dispatch_view(ctypes.byref(cfg), _p(ws), _nbytes(ws),
                                           *[ctypes.byref(p) for p in ptrs]), True)
    E, T, k = cfg.n_experts, cfg.T, cfg.top_k
    out = []
    for p, n in zip(ptrs, (E + 1, T * k, T * k)):
        off = int(p.value) - ws.data_ptr()
        out.append(ws[off:off + 4 * n].view(torch.int32))
    return out[0], out[1].view(T, k), out[2]


def moe_backward_workspace_size(cfg: MoEConfig) -> int:
    return int(lib().moe_backward_workspace_size(ctypes.byref(cfg)))


def moe_backward(cfg, x, w_router, logit_offset, weights: Dict, topk_idx, topk_w, dout, dx,
                 dw_router, grads: Dict, fws, bws, stream=None, check=True) -> int:
    """Backward of the layer after moe_forward ran with workspace ``fws``;
    ``grads`` maps dw1, dw3, dw2 (and dws1, dws3, dws2) to output tensors."""
    w = expert_weights(weights)
    g = MoEExpertGrads(*[_p(grads.get(n)) for n in ("dw1", "dw3", "dw2", "dws1", "dws3",
                                                      "dws2")])
    st = lib().moe_backward(ctypes.byref(cfg), _p(x), _p(w_router), _p(logit_offset),
                            ctypes.byref(w), _p(topk_idx), _p(topk_w), _p(dout), _p(dx),
                            _p(dw_router), ctypes.byref(g), _p(fws), _nbytes(fws), _p(bws),
                            _nbytes(bws), _s(stream))
    return _check(st, check)


FORWARD_PHASES = 6


def moe_forward_profiled(cfg, x, w_router, sel_bias, logit_offset, weights: Dict, out, topk_idx,
                         topk_w, counts, ws, events, stream=None, check=True) -> int:
    """``events``: FORWARD_PHASES + 1 torch.cuda.Event objects (timing enabled)."""
    w = expert_weights(weights)
    for e in events:
        if e.cuda_event == 0:      # torch creates the CUDA event on first record
            e.record()
    arr = (ctypes.c_void_p * (FORWARD_PHASES + 1))(*[e.cuda_event for e in events])
    st = lib().moe_forward_profiled(ctypes.byref(cfg), _p(x), _p(w_router), _p(sel_bias),
                                    _p(logit_offset), ctypes.byref(w), _p(out), _p(topk_idx),
                                    _p(topk_w), _p(counts), _p(ws),
                                    _nbytes(ws) if ws is not None else 0, _s(stream), arr)
    return _check(st, check)


def moe_device_status(ws, stream=None):
    """(status, raw flag bits); synchronises the stream."""
    flags = ctypes.c_uint32(0)
    st = lib().moe_device_status(_p(ws), _nbytes(ws), _s(stream), ctypes.byref(flags))
    return int(st), int(flags.value)


def moe_router_refined_tokens(ws, stream=None) -> int:
    """Tokens the last bf16 router call re-decided on exact logits (synchronises)."""
    c = ctypes.c_int32(0)
    _check(lib().moe_router_refined_tokens(_p(ws), _nbytes(ws), _s(stream), ctypes.byref(c)), True)
    return int(c.value)


def moe_selftest_bounded_wait(ws, limit_seconds=0.05, stream=None, check=True) -> int:
    """Run the bounded-wait self-test kernel (returns after limit_seconds)."""
    st = lib().moe_selftest_bounded_wait(_p(ws), _nbytes(ws), float(limit_seconds), _s(stream))
    return _check(st, check)
