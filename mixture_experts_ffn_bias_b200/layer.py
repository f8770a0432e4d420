"""Device-side buffers for one MoE layer and calls into the C ABI.

PyTorch supplies device memory and streams only; every step of the layer runs
in libmoe_b200.so.  ``MoELayer`` uploads a workload's host arrays (as produced
by :mod:`.inputs`), owns the output buffers and the workspace, and exposes the
calls of the ABI with those buffers filled in.
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np
import torch

from . import binding as B
from .inputs import DTYPE_BF16, MoEShape

_WEIGHT_KEYS = ("w1", "w3", "w2", "ws1", "ws3", "ws2")


def act_dtype(shape: MoEShape) -> torch.dtype:
    return torch.bfloat16 if shape.dtype == DTYPE_BF16 else torch.float32


def to_device(a: np.ndarray, dtype: torch.dtype, device) -> torch.Tensor:
    """Host float32 array (bf16-exact for bf16) -> contiguous device tensor."""
    t = torch.from_numpy(np.ascontiguousarray(a)).to(device=device)
    return t.to(dtype).contiguous()


class MoELayer:
    def __init__(self, shape: MoEShape, host: Dict[str, np.ndarray], device="cuda"):
        self.shape = shape
        self.device = torch.device(device)
        self.cfg = B.config_from_shape(shape)
        st = B.moe_check_config(self.cfg)
        if st != B.MOE_OK:
            raise B.MoEError(st, "configuration rejected: " + B.status_string(st))
        dt = act_dtype(shape)
        self.dtype = dt
        self.x = to_device(host["x"], dt, self.device)
        self.w_router = to_device(host["w_router"], dt, self.device)
        self.weights = {k: to_device(host[k], dt, self.device) for k in _WEIGHT_KEYS if k in host}
        self.sel_bias = (to_device(host["sel_bias"], torch.float32, self.device)
                         if "sel_bias" in host else None)
        self.logit_offset = (to_device(host["logit_offset"], torch.float32, self.device)
                             if "logit_offset" in host else None)
        T, d, E, k = shape.T, shape.d_model, shape.n_experts, shape.top_k
        kw = dict(device=self.device)
        self.out = torch.empty((T, d), dtype=dt, **kw)
        self.topk_idx = torch.empty((T, k), dtype=torch.int32, **kw)
        self.topk_w = torch.empty((T, k), dtype=torch.float32, **kw)
        self.counts = torch.empty((E,), dtype=torch.int32, **kw)
        self.ws = torch.empty((max(B.moe_workspace_size(self.cfg), 256),), dtype=torch.uint8, **kw)

    # ----------------------------------------------------------------- calls
    def forward(self, x: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                stream=None, gather_rows: bool = False, fold_combine: bool = False,
                scatter_in_gemm: bool = False) -> torch.Tensor:
        """The layer forward (moe_forward; moe_forward_ex with gather_rows,
        fold_combine or scatter_in_gemm)."""
        args = (self.cfg, self.x if x is None else x, self.w_router, self.sel_bias,
                self.logit_offset, self.weights, self.out if out is None else out,
                self.topk_idx, self.topk_w, self.counts, self.ws)
        if gather_rows or fold_combine or scatter_in_gemm:
            B.moe_forward_ex(*args, gather_rows=int(gather_rows),
                             fold_combine=int(fold_combine),
                             scatter_in_gemm=int(scatter_in_gemm), stream=stream)
        else:
            B.moe_forward(*args, stream=stream)
        return self.out if out is None else out

    def dispatch_view(self):
        """(offsets, slot_pos, perm_src) of the last forward, read from the
        workspace (int32 device views; valid until the next call on it)."""
        return B.moe_forward_dispatch_view(self.cfg, self.ws)

    def backward(self, dout: torch.Tensor, stream=None) -> Dict[str, torch.Tensor]:
        """Gradients of <dout, out> for the last forward (bf16 layers): dx,
        dw_router (fp32) and dw1, dw3, dw2 (and the shared expert's)."""
        if not hasattr(self, "bws"):
            n = B.moe_backward_workspace_size(self.cfg)
            if n == 0:
                raise B.MoEError(B.MOE_ERR_UNSUPPORTED, "backward needs a bf16 layer")
            self.bws = torch.empty((n,), dtype=torch.uint8, device=self.device)
        g = {"dx": torch.empty_like(self.x),
             "dw_router": torch.empty(self.w_router.shape, dtype=torch.float32,
                                      device=self.device)}
        for k, v in self.weights.items():
            g["d" + k] = torch.empty_like(v)
        B.moe_backward(self.cfg, self.x, self.w_router, self.logit_offset, self.weights,
                       self.topk_idx, self.topk_w, dout, g["dx"], g["dw_router"], g, self.ws,
                       self.bws, stream)
        return g

    def bias_update(self, counts: Optional[torch.Tensor] = None, rate=1e-3, starved_frac=0.1,
                    starved_add=0.5, clamp=10.0, stream=None):
        if self.sel_bias is None:
            self.sel_bias = torch.zeros(self.shape.n_experts, dtype=torch.float32,
                                        device=self.device)
        B.moe_bias_update(self.cfg, self.counts if counts is None else counts, self.sel_bias,
                          rate, starved_frac, starved_add, clamp, stream)

    def device_status(self, stream=None):
        return B.moe_device_status(self.ws, stream)
