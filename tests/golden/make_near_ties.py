"""Writes near_ties.json: for every workload, the tokens the layer's parity
bar excludes from the bit-exact routing comparison.

A token is excluded when the oracle's fp64 selection keys of its k-th and
(k+1)-th picks differ by less than 1e-6 (at such a gap the fp32 router may
legitimately order them the other way).  Only the oracle and the seeded
input generator are called, so the stored counts never come from the CUDA
path.

    python tests/golden/make_near_ties.py      # rewrites near_ties.json
"""
from __future__ import annotations

import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

from mixture_experts_ffn_bias_b200 import inputs as I  # noqa: E402
from oracle import moe_oracle as O  # noqa: E402

NEAR_TIE = 1e-6
OUT = os.path.join(HERE, "near_ties.json")


def near_ties(shape) -> dict:
    host = I.make_inputs(shape)
    r = O.router(host["x"], host["w_router"], shape.top_k, shape.gate,
                 bool(shape.norm_topk_prob), host.get("sel_bias"), host.get("logit_offset"))
    excluded = r.edge_gap < NEAR_TIE
    return {"T": shape.T, "excluded": int(excluded.sum()),
            "tokens": [int(t) for t in excluded.nonzero()[0]]}


def main():
    table = {"rule": "oracle fp64 key_(k) - key_(k+1) < 1e-6", "workloads": {}}
    for name in I.WORKLOAD_ORDER:
        table["workloads"][name] = near_ties(I.WORKLOADS[name])
        print(name, table["workloads"][name]["excluded"], flush=True)
    with open(OUT, "w") as f:
        json.dump(table, f, indent=1)
        f.write("\n")


if __name__ == "__main__":
    main()
