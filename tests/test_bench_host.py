"""Host arithmetic of bench.py's JSON line (no GPU): the algorithmic FLOPs
the roofline divides by, and when a captured DRAM traffic figure may be
reported."""
import hashlib
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from mixture_experts_ffn_bias_b200 import inputs as I  # noqa: E402


def test_gateup_launch_flops_counts_the_shared_group_in_the_same_launch():
    q = I.WORKLOADS["qwen3_30b"]      # no shared expert: 4 R d F
    assert bench.gateup_launch_flops(q) == 4 * 16384 * 8 * 2048 * 768
    p = I.WORKLOADS["page2"]          # routed 4 R d F + shared 4 T d Fs
    assert bench.gateup_launch_flops(p) == 4 * 8192 * 2 * 640 * 1024 + 4 * 8192 * 640 * 1024
    t = I.WORKLOADS["tiny"]           # fp32: the shared expert has launches of its own
    assert bench.gateup_launch_flops(t) == 4 * t.T * t.top_k * t.d_model * t.d_ff


def _sha():
    src = os.path.join(ROOT, "mixture_experts_ffn_bias_b200", "csrc", "grouped_gemm_sm100.cu")
    with open(src, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def test_captured_traffic_is_reported_only_for_the_captured_source(monkeypatch):
    q = I.WORKLOADS["qwen3_30b"]
    monkeypatch.setattr(bench, "GATEUP_TRAFFIC", {"qwen3_30b": (123, _sha())})
    nbytes, note = bench.gateup_traffic(q)
    assert nbytes == 123 and "not measured in this run" in note
    monkeypatch.setattr(bench, "GATEUP_TRAFFIC", {"qwen3_30b": (123, "0" * 16)})
    nbytes, note = bench.gateup_traffic(q)
    assert nbytes is None and "not reported" in note
    assert bench.gateup_traffic(I.WORKLOADS["page2"])[0] is None
