"""Seeded synthetic inputs for the MoE FFN layer.

This module only draws numbers and rounds them to the storage dtype; it holds
none of the layer's arithmetic, so both the CUDA path and the CPU oracle can
read the same bytes from it without sharing any of the method.

Workloads (shapes of the models on the pages):

* ``tiny``       T=256,   d=64,   E=4   routed, F=128,  top-2, softmax+renorm, fp32
* ``page2``      T=8192,  d=640,  E=16  routed + 1 shared, F=1024, top-2, sigmoid,
                 fp32 selection bias ~ U(-0.5, 0.5)  (moe-200m-qwen3-100b README,
                 "Resulting architecture" and ``MoEModelConfig``)
* ``qwen3_30b``  T=16384, d=2048, E=128 routed, F=768, top-8, softmax+norm_topk_prob
                 (SpecForge PR #930, "qwen3 MoE preset"; Qwen3-30B-A3B-like shape)
* ``wide``       T=4096,  d=5120, E=16 routed, F=4352, top-4, softmax+renorm, fp32
                 selection bias ~ U(-0.5, 0.5) (SpecForge PR #930, 16x4352 top-4 arm)
* ``skew``       T=32768, d=2048, E=64 routed + 1 shared, F=1024, top-6, sigmoid,
                 Zipf(s=1.2) per-expert logit offsets, bias 0 then one update
                 (SpecForge PR #931, 64-expert top-6 arm and its routing collapse)

Draw order per workload (``numpy.random.default_rng(seed)``): x, w_router, w1, w3,
w2, [ws1, ws3, ws2], sel_bias, expert permutation for the Zipf offsets.
x ~ N(0,1); every weight ~ N(0, 0.02); bf16 workloads round each value to
bf16 (round to nearest even) and keep it as a float32 array holding exactly
that bf16 value.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import numpy as np

GATE_SOFTMAX = 0
GATE_SIGMOID = 1
DTYPE_F32 = 0
DTYPE_BF16 = 1


@dataclasses.dataclass(frozen=True)
class MoEShape:
    name: str
    T: int                 # tokens
    d_model: int
    n_experts: int         # routed experts E
    d_ff: int              # routed expert width F
    top_k: int
    n_shared: int          # 0 or 1 shared expert
    d_ff_shared: int
    gate: int              # GATE_SOFTMAX / GATE_SIGMOID
    norm_topk_prob: int    # renormalise the top-k combine weights
    dtype: int             # DTYPE_F32 / DTYPE_BF16 (activations and weights)
    bias: str              # "none" | "uniform" | "zero"
    zipf_s: float          # 0 = no per-expert logit offsets
    seed: int

    def replace(self, **kw) -> "MoEShape":
        return dataclasses.replace(self, **kw)

    @property
    def rows(self) -> int:
        """Routed rows R = T * k."""
        return self.T * self.top_k


WORKLOADS: Dict[str, MoEShape] = {
    "tiny": MoEShape("tiny", 256, 64, 4, 128, 2, 0, 0, GATE_SOFTMAX, 1,
                     DTYPE_F32, "none", 0.0, 0),
    "page2": MoEShape("page2", 8192, 640, 16, 1024, 2, 1, 1024, GATE_SIGMOID, 1,
                      DTYPE_BF16, "uniform", 0.0, 1),
    "qwen3_30b": MoEShape("qwen3_30b", 16384, 2048, 128, 768, 8, 0, 0,
                          GATE_SOFTMAX, 1, DTYPE_BF16, "none", 0.0, 2),
    "wide": MoEShape("wide", 4096, 5120, 16, 4352, 4, 0, 0, GATE_SOFTMAX, 1,
                     DTYPE_BF16, "uniform", 0.0, 3),
    "skew": MoEShape("skew", 32768, 2048, 64, 1024, 6, 1, 1024, GATE_SIGMOID, 1,
                     DTYPE_BF16, "zero", 1.2, 4),
}
WORKLOAD_ORDER = ["tiny", "page2", "qwen3_30b", "wide", "skew"]


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); return float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Upper 16 bits of float32 values that are already bf16-exact."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    return (a.view(np.uint32) >> 16).astype(np.uint16)


def _normal(rng: np.random.Generator, shape, std: float, bf16: bool) -> np.ndarray:
    a = rng.standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return round_to_bf16(a) if bf16 else a


def make_inputs(shape: MoEShape, seed: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Draw one workload's tensors (host float32 arrays, bf16-exact when bf16)."""
    rng = np.random.default_rng(shape.seed if seed is None else seed)
    bf16 = shape.dtype == DTYPE_BF16
    T, d, E, F, k = shape.T, shape.d_model, shape.n_experts, shape.d_ff, shape.top_k
    out: Dict[str, np.ndarray] = {}
    out["x"] = _normal(rng, (T, d), 1.0, bf16)
    out["w_router"] = _normal(rng, (E, d), 0.02, bf16)
    out["w1"] = _normal(rng, (E, F, d), 0.02, bf16)      # gate projection [E, out, in]
    out["w3"] = _normal(rng, (E, F, d), 0.02, bf16)      # up projection   [E, out, in]
    out["w2"] = _normal(rng, (E, d, F), 0.02, bf16)      # down projection [E, out, in]
    if shape.n_shared:
        Fs = shape.d_ff_shared
        out["ws1"] = _normal(rng, (Fs, d), 0.02, bf16)
        out["ws3"] = _normal(rng, (Fs, d), 0.02, bf16)
        out["ws2"] = _normal(rng, (d, Fs), 0.02, bf16)
    if shape.bias == "uniform":
        out["sel_bias"] = rng.uniform(-0.5, 0.5, size=E).astype(np.float32)
    elif shape.bias == "zero":
        out["sel_bias"] = np.zeros(E, dtype=np.float32)
    if shape.zipf_s > 0.0:
        perm = rng.permutation(E)
        off = np.empty(E, dtype=np.float32)
        for r in range(1, E + 1):
            off[perm[r - 1]] = np.float32(-shape.zipf_s * math.log(r))
        out["logit_offset"] = off
    return out


def make_tokens(shape: MoEShape, seed: int) -> np.ndarray:
    """A fresh batch of activations x[T, d] for the same layer (x ~ N(0,1))."""
    rng = np.random.default_rng(seed)
    return _normal(rng, (shape.T, shape.d_model), 1.0, shape.dtype == DTYPE_BF16)
