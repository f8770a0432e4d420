#!/usr/bin/env python
"""MoE FFN layer forward on B200: tokens/s and grouped-GEMM TFLOP/s.

One step = one pass of the whole layer path on one batch: router, dispatch,
grouped SwiGLU experts (+ shared expert), combine, then the per-expert counts
are summed over data-parallel ranks (NCCL all-reduce, N > 1 only) and the
selection-bias update runs.  Each rank holds a full replica of the layer and
its own T tokens (weak scaling); ``value`` is the tokens of all ranks per
second, timed on the device (CUDA events, max over ranks).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...     # the CPU oracle, timed on host cores

With --gpus N > 1 and no torchrun environment, the script re-launches itself
under torch.distributed.run with N ranks (one per GPU, NCCL).  Prints one
JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import json
import os
import socket
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mixture_experts_ffn_bias_b200 import inputs as I  # noqa: E402

METRIC = "MoE-layer fwd tokens/sec and grouped-GEMM TFLOP/s (% bf16 peak) on 1 B200"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NOMINAL_BF16_TFLOPS = 2250.0      # B200 dense bf16, NVIDIA's nominal figure
L2_BYTES = 126 * 1024 * 1024


# --------------------------------------------------------------------------- #
# workload arithmetic                                                          #
# --------------------------------------------------------------------------- #
def layer_flops(s: I.MoEShape) -> dict:
    R = s.T * s.top_k
    return {
        "router": 2 * s.T * s.d_model * s.n_experts,
        "gate_up": 4 * R * s.d_model * s.d_ff,
        "down": 2 * R * s.d_ff * s.d_model,
        "shared": 6 * s.T * s.d_model * s.d_ff_shared * s.n_shared,
    }


def gateup_launch_flops(s: I.MoEShape) -> int:
    """Algorithmic FLOPs of one gate/up GEMM launch: the routed experts'
    4 R d F, plus the shared expert's 4 T d Fs on bf16 layers, whose gate/up
    runs as one more group of the same launch."""
    fl = layer_flops(s)["gate_up"]
    if s.dtype == I.DTYPE_BF16:
        fl += 4 * s.T * s.d_model * s.d_ff_shared * s.n_shared
    return fl


# DRAM bytes per launch of the routed gate/up GEMM, from the ncu capture in
# profiles/grouped_gemm_gateup_qwen3_30b.md, and the kernel source it was
# taken on (sha256 of csrc/grouped_gemm_sm100.cu, first 16 hex digits).
GATEUP_TRAFFIC = {"qwen3_30b": (2154375424, "0a08a2e8d9e85551")}


def gateup_traffic(s: I.MoEShape):
    """(DRAM bytes per gate/up launch or None, note): the bytes of the ncu
    capture when it was taken on the kernel source in the tree, else None."""
    import hashlib
    src = os.path.join(ROOT, "mixture_experts_ffn_bias_b200", "csrc", "grouped_gemm_sm100.cu")
    with open(src, "rb") as f:
        sha = hashlib.sha256(f.read()).hexdigest()[:16]
    if s.name not in GATEUP_TRAFFIC:
        return None, "not measured: no ncu capture of this workload's gate/up launch"
    nbytes, at = GATEUP_TRAFFIC[s.name]
    where = ("ncu capture (dram__bytes_read.sum + dram__bytes_write.sum, one launch) in "
             "profiles/grouped_gemm_gateup_qwen3_30b.md")
    if sha != at:
        return None, (f"{nbytes} DRAM bytes per launch in the {where}, taken on kernel source "
                      f"{at}; the source is now {sha}, so not reported")
    return nbytes, f"from the {where}, on this kernel source ({sha}); not measured in this run"


def near_tie_exclusions(s: I.MoEShape) -> dict:
    """Tokens the parity bar excludes on this workload (the oracle's k-th and
    (k+1)-th selection keys closer than 1e-6), as counted by
    tests/golden/make_near_ties.py from the oracle; the GPU tests compare
    every other token bit for bit."""
    path = os.path.join(ROOT, "tests", "golden", "near_ties.json")
    try:
        with open(path) as f:
            g = json.load(f)
        w = g["workloads"][s.name]
        if w["T"] != s.T:
            return {"count": None, "note": f"counted at T={w['T']}, this run has T={s.T}"}
        return {"count": w["excluded"], "of_tokens": w["T"], "rule": g["rule"],
                "source": "tests/golden/near_ties.json"}
    except (OSError, KeyError, ValueError):
        return {"count": None, "note": "not counted for this workload"}


def describe(s: I.MoEShape) -> str:
    gate = "softmax" if s.gate == I.GATE_SOFTMAX else "sigmoid"
    dt = "bf16" if s.dtype == I.DTYPE_BF16 else "fp32"
    sh = f" + {s.n_shared} shared (F={s.d_ff_shared})" if s.n_shared else ""
    return (f"{s.name}: T={s.T} d_model={s.d_model} E={s.n_experts} routed (F={s.d_ff}){sh} "
            f"top-{s.top_k} {gate}{'+renorm' if s.norm_topk_prob else ''} {dt}")


def load_peaks() -> tuple:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def step_bytes(s: I.MoEShape) -> int:
    """Bytes one forward step touches at least once: weights, x, the
    permuted rows, h, the expert outputs and out."""
    b = 2 if s.dtype == I.DTYPE_BF16 else 4
    R = s.T * s.top_k
    w = (3 * s.n_experts * s.d_ff * s.d_model + s.n_experts * s.d_model
         + 3 * s.n_shared * s.d_ff_shared * s.d_model) * b
    act = (2 * s.T * s.d_model + 2 * R * s.d_model + R * s.d_ff
           + s.n_shared * s.T * (s.d_ff_shared + s.d_model)) * b
    return w + act


def host_cpu() -> dict:
    model = ""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"host_cores": len(os.sched_getaffinity(0)), "cpu_model": model}


# --------------------------------------------------------------------------- #
# clocks during the timed region                                              #
# --------------------------------------------------------------------------- #
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != 6:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[2:]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------------- #
# CPU oracle (baseline and reference arm)                                      #
# --------------------------------------------------------------------------- #
def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


class OracleRunner:
    """The oracle as it stands, on windows of the workload's tokens.  Weights
    are handed to it already widened to float64 (same values), so a window's
    cost is its own arithmetic."""

    def __init__(self, shape: I.MoEShape, host: dict):
        from oracle import moe_oracle as O
        self.O = O
        self.shape = shape
        self.host = {k: (v.astype(np.float64) if k != "x" else v) for k, v in host.items()}
        self.pos = 0

    def run(self, n: int) -> float:
        s = self.shape
        lo = self.pos % s.T
        hi = min(lo + n, s.T)
        self.pos = hi
        win = dict(self.host)
        win["x"] = self.host["x"][lo:hi]
        t0 = time.perf_counter()
        r = self.O.router(win["x"], win["w_router"], s.top_k, s.gate, bool(s.norm_topk_prob),
                          win.get("sel_bias"), win.get("logit_offset"))
        self.O.dispatch(r.topk_idx, s.n_experts)
        self.O.moe_forward(win, s.top_k, s.gate, bool(s.norm_topk_prob), routing=r)
        return time.perf_counter() - t0, hi - lo

    def calibrate(self, seconds: float) -> int:
        """Tokens per window so that one window takes about `seconds`."""
        n = 16
        for _ in range(6):
            t, m = self.run(n)
            if t >= 0.5 * seconds or n >= self.shape.T:
                break
            n = min(self.shape.T, max(n + 1, int(n * min(8.0, seconds / max(t, 1e-3)))))
        return max(1, min(self.shape.T, int(n * seconds / max(t, 1e-3))))


def cpu_baseline(shape, host, seconds=15.0) -> dict:
    runner = OracleRunner(shape, host)
    n = runner.calibrate(seconds / 3)
    t, m = runner.run(n)
    tot_t, tot_m = t, m
    while tot_t < seconds and m > 0:
        t, m = runner.run(n)
        tot_t += t
        tot_m += m
    return {"value": tot_m / tot_t, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"{tot_m} of the workload's tokens in windows of {n}: router, dispatch, "
                      f"{shape.n_experts} experts{' + shared' if shape.n_shared else ''}, "
                      f"combine, fp64 numpy ({tot_t:.1f} s)", **host_cpu()}


def run_reference(args, shape, rank: int, world: int):
    if rank != 0:
        return
    host = I.make_inputs(shape)
    runner = OracleRunner(shape, host)
    budget = 150.0 / max(1, args.steps + args.warmup)
    n = runner.calibrate(budget)
    for _ in range(args.warmup):
        runner.run(n)
    ts, ms = 0.0, 0
    for _ in range(args.steps):
        t, m = runner.run(n)
        ts += t
        ms += m
    value = ms / ts
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * ts / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": describe(shape), "parallelism": "host cores"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(),
                         "kind": "oracle",
                         "sample": f"{n} tokens per step (of {shape.T}), full layer in fp64",
                         **host_cpu()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- #
# GPU arm                                                                      #
# --------------------------------------------------------------------------- #
def run_backward(args, shape):
    """--mode backward (one GPU): moe_backward after a forward, timed with
    CUDA events over --steps calls after --warmup calls.  The expert GEMM
    FLOPs of a backward are 16 R d F (+ 16 T d Fs for a shared expert):
    dH, the recomputed G and U, dX (K = 2F) and the three weight gradients."""
    import numpy as np
    import torch
    from mixture_experts_ffn_bias_b200 import binding as B
    from mixture_experts_ffn_bias_b200.layer import MoELayer, to_device

    dev = torch.device("cuda", 0)
    host = I.make_inputs(shape)
    layer = MoELayer(shape, host, dev)
    if layer.sel_bias is None:
        layer.sel_bias = torch.zeros(shape.n_experts, dtype=torch.float32, device=dev)
    dout = to_device(I.round_to_bf16(np.random.default_rng(shape.seed + 77).standard_normal(
        (shape.T, shape.d_model)).astype(np.float32)), torch.bfloat16, dev)
    layer.forward()
    for _ in range(args.warmup):
        layer.backward(dout)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        layer.backward(dout)
    e1.record()
    torch.cuda.synchronize(dev)
    st, flags = B.moe_device_status(layer.bws)
    if st != B.MOE_OK:
        raise SystemExit(f"device status after the backward: {B.status_string(st)} ({flags})")
    ms = e0.elapsed_time(e1) / args.steps
    R = shape.T * shape.top_k
    fl = 16.0 * R * shape.d_model * shape.d_ff
    if shape.n_shared:
        fl += 16.0 * shape.T * shape.d_model * shape.d_ff_shared
    peaks, kind = load_peaks()
    sus = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    tf = fl / (ms * 1e-3) / 1e12
    print(json.dumps({
        "metric": "MoE-layer backward tokens/sec (moe_backward after moe_forward) on 1 B200",
        "value": shape.T / (ms * 1e-3), "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "dtype": "bf16",
        "data": "synthetic", "config": {"workload": describe(shape)},
        "expert_gemm": {"tflops": tf, "frac_of_sustained": tf / sus,
                        "peaks": kind, "flops_per_step": fl},
        "workspace_gb": layer.bws.numel() / 1e9}), flush=True)


def path_bytes(s: I.MoEShape) -> dict:
    """Algorithmic bytes of the HBM-bound steps: the router reads x and the
    router weight and writes the routing; dispatch reads x once and writes
    the permuted rows; the combine reads the expert rows (and the shared
    expert's output) and writes out.  Each tensor counted once per step that
    reads or writes it."""
    b = 2 if s.dtype == I.DTYPE_BF16 else 4
    R = s.T * s.top_k
    return {
        "router": s.T * s.d_model * b + s.n_experts * s.d_model * b + s.T * s.top_k * 8,
        "dispatch": s.T * s.d_model * b + R * s.d_model * b + R * 8,
        "combine": R * s.d_model * b + R * 8 + s.n_shared * s.T * s.d_model * b
        + s.T * s.d_model * b,
    }


def run_ours(args, shape, rank: int, world: int, local_rank: int):
    import torch
    import torch.distributed as dist
    from mixture_experts_ffn_bias_b200 import binding as B
    from mixture_experts_ffn_bias_b200.dp import allreduce_counts
    from mixture_experts_ffn_bias_b200.layer import MoELayer

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    host = I.make_inputs(shape)
    if rank > 0:
        host["x"] = I.make_tokens(shape, seed=1000 * (shape.seed + 1) + rank)
    layer = MoELayer(shape, host, dev)
    if layer.sel_bias is None:
        layer.sel_bias = torch.zeros(shape.n_experts, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    nph = B.FORWARD_PHASES
    # A step whose data fits a few times in L2 would be timed warm: write a
    # buffer larger than L2 before every timed step instead.
    flush = args.l2_flush == "on" or (args.l2_flush == "auto" and step_bytes(shape) < 4 * L2_BYTES)
    flush_buf = torch.empty(4 * L2_BYTES, dtype=torch.uint8, device=dev) if flush else None

    def step(evs=None, x=None, out=None):
        if evs is None:
            layer.forward(x=x, out=out)
        else:
            B.moe_forward_profiled(layer.cfg, layer.x if x is None else x, layer.w_router,
                                   layer.sel_bias, layer.logit_offset, layer.weights, layer.out,
                                   layer.topk_idx, layer.topk_w, layer.counts, layer.ws, evs)
        allreduce_counts(layer.counts)
        layer.bias_update()

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        if flush:
            flush_buf.fill_(1)
        step()
    st, flags = layer.device_status()
    if st != B.MOE_OK:
        raise SystemExit(f"device status after warm-up: {B.status_string(st)} ({flags})")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nph + 1)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    per = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)] if flush else []
    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler(f"GPU-{props.uuid}" if getattr(props, "uuid", None) else str(local_rank))
    barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    start.record(stream)
    for i in range(args.steps):
        if flush:
            flush_buf.fill_(i & 0xff)
            per[i][0].record(stream)
        step()
        if flush:
            per[i][1].record(stream)
    end.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    barrier()
    t_ms = (sum(a.elapsed_time(b) for a, b in per) if flush else start.elapsed_time(end))
    # Per-phase times come from separate steps with events between the
    # phases: an event breaks the early launch of the kernel after it, so
    # the timed steps above run without them.
    for i in range(args.steps):
        if flush:
            flush_buf.fill_(i & 0xff)
        step(evs[i])
    torch.cuda.synchronize(dev)
    barrier()
    phases = [statistics.mean(evs[i][p].elapsed_time(evs[i][p + 1]) for i in range(args.steps))
              for p in range(nph)]
    st, flags = layer.device_status()
    if st != B.MOE_OK:
        raise SystemExit(f"device status after timing: {B.status_string(st)} ({flags})")
    refined = B.moe_router_refined_tokens(layer.ws)

    # End to end through the public layer call: every step copies its x in
    # from pinned host memory and its output back.  Two buffers each way and
    # one copy stream per direction, so step i's copies overlap the compute
    # of its neighbours (both directions of the link at once).
    e2e_steps = max(3, min(args.steps, 50))
    x_host = layer.x.to("cpu").pin_memory()
    out_host = [torch.empty(layer.out.shape, dtype=layer.out.dtype).pin_memory() for _ in range(2)]
    x_dev = [torch.empty_like(layer.x) for _ in range(2)]
    out_dev = [torch.empty_like(layer.out) for _ in range(2)]
    h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    h2d_done, comp_done, d2h_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    e0.record(stream)
    h2d.wait_event(e0)
    d2h.wait_event(e0)
    with torch.cuda.stream(h2d):
        x_dev[0].copy_(x_host, non_blocking=True)
        h2d_done[0].record(h2d)
    for i in range(e2e_steps):
        b = i & 1
        stream.wait_event(h2d_done[b])
        if i >= 2:
            stream.wait_event(d2h_done[b])          # out_dev[b] read out by then
        step(x=x_dev[b], out=out_dev[b])
        comp_done[b].record(stream)
        if i + 1 < e2e_steps:
            with torch.cuda.stream(h2d):
                if i >= 1:
                    h2d.wait_event(comp_done[1 - b])  # step i-1 done with x_dev[1-b]
                x_dev[1 - b].copy_(x_host, non_blocking=True)
                h2d_done[1 - b].record(h2d)
        with torch.cuda.stream(d2h):
            d2h.wait_event(comp_done[b])
            out_host[b].copy_(out_dev[b], non_blocking=True)
            d2h_done[b].record(d2h)
    for b in range(min(2, e2e_steps)):
        stream.wait_event(d2h_done[b])
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps

    if world > 1:
        t = torch.tensor([t_ms, e2e_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        t_ms, e2e_ms = float(t[0]), float(t[1])

    if rank == 0:
        ms = t_ms / args.steps
        fl = layer_flops(shape)
        peaks, peak_kind = load_peaks()
        sus = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
        burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
        hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        t_gateup = phases[2] * 1e-3
        t_gemm = (phases[2] + phases[3] + phases[4]) * 1e-3
        launch_flops = gateup_launch_flops(shape)
        achieved = launch_flops / t_gateup / 1e12
        traffic = gateup_traffic(shape)
        gemm_tflops = (fl["gate_up"] + fl["down"] + fl["shared"]) / t_gemm / 1e12
        pb = path_bytes(shape)
        t_path = (phases[0] + phases[1] + phases[5]) * 1e-3
        path_gbs = sum(pb.values()) / t_path / 1e9
        # router 2 (bf16: tensor-core router + refine; fp32: logits + select),
        # dispatch 2 (rank with the scan, scatter), experts 2 (bf16: the shared
        # expert runs inside the routed launches; fp32: 2 more for it),
        # combine 1, bias update 1
        shared_launches = 0 if shape.dtype == I.DTYPE_BF16 else 2 * shape.n_shared
        per_step_launches = 2 + 2 + 2 + shared_launches + 1 + 1
        l2 = ("flushed: a 504 MB buffer is written before every timed step (the step's data "
              "would fit in L2)" if flush else
              f"not flushed: each step streams {step_bytes(shape) / 1e9:.2f} GB (weights + "
              "activations) through the 126 MB L2")
        line = {
            "metric": METRIC, "value": shape.T * world / (ms * 1e-3), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16"
            if shape.dtype == I.DTYPE_BF16 else "f32", "data": "synthetic",
            "config": {"workload": describe(shape), "tokens_per_gpu": shape.T,
                       "parallelism": f"dp{world} (replicated layer, counts all-reduce)",
                       "l2": l2},
            "grouped_gemm": {"tflops": gemm_tflops, "frac_of_burst": gemm_tflops / burst,
                             "frac_of_sustained": gemm_tflops / sus,
                             "frac_of_nominal": gemm_tflops / NOMINAL_BF16_TFLOPS,
                             "peaks": peak_kind},
            "routing_permute_combine": {"bytes": sum(pb.values()), "ms": t_path * 1e3,
                                        "gbs": path_gbs, "frac_of_hbm": path_gbs / hbm,
                                        "peaks": peak_kind},
            "phases_ms": dict(zip(["router", "dispatch", "gate_up", "down", "shared", "combine"],
                                  phases)),
            "roofline": {"kernel": "grouped gate/up GEMM + SwiGLU (tcgen05)" +
                         (", shared expert as one more group"
                          if shape.n_shared and shape.dtype == I.DTYPE_BF16 else ""),
                         "bound": "tensor", "flops_per_launch": launch_flops,
                         "achieved": achieved, "peak": burst, "unit": "TFLOP/s",
                         "frac": achieved / burst,
                         "peak_kind": f"bf16_tflops, burst ({peak_kind})",
                         "frac_of_sustained": achieved / sus,
                         "frac_of_nominal": achieved / NOMINAL_BF16_TFLOPS,
                         "traffic": traffic[0],
                         "traffic_note": traffic[1]},
            "e2e": {"value": shape.T * world / (e2e_ms * 1e-3), "unit": UNIT,
                    "h2d_bytes_per_step": layer.x.numel() * layer.x.element_size(),
                    "d2h_bytes_per_step": layer.out.numel() * layer.out.element_size(),
                    "copies": "pinned host, one cudaMemcpyAsync per tensor per step, "
                              "double-buffered on two copy streams"},
            "router_refined_tokens_last_step": refined,
            "near_tie_exclusions": near_tie_exclusions(shape),
            "gpu_launches": per_step_launches * args.steps,
            "clocks": clocks,
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(shape, host)
        print(json.dumps(line), flush=True)


def check_ranks(args, rank: int, world: int, local_rank: int):
    """--check-ranks: the multi-rank plumbing alone.  Every rank sums a
    per-expert count vector with the others (NCCL on GPUs, gloo without
    one); rank 0 prints the world size and whether the sum came out right."""
    import datetime

    import torch
    import torch.distributed as dist
    from mixture_experts_ffn_bias_b200.dp import allreduce_counts

    cuda = torch.cuda.is_available()
    if world > 1:
        kw = {}
        if cuda:
            torch.cuda.set_device(local_rank)
            kw["device_id"] = torch.device("cuda", local_rank)
        dist.init_process_group("nccl" if cuda else "gloo",
                                timeout=datetime.timedelta(seconds=60), **kw)
    dev = torch.device("cuda", local_rank) if cuda else torch.device("cpu")
    try:
        counts = torch.full((8,), rank + 1, dtype=torch.int32, device=dev)
        allreduce_counts(counts)
        ok = bool((counts == world * (world + 1) // 2).all())
        if rank == 0:
            print(json.dumps({"check": "ranks", "n_gpus": args.gpus, "world_size": world,
                              "backend": dist.get_backend() if world > 1 else None,
                              "counts_allreduce_ok": ok}), flush=True)
        if not ok:
            raise SystemExit("counts all-reduce gave a wrong sum")
    finally:
        if world > 1:
            dist.destroy_process_group()


def free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def relaunch_command(argv, n: int, port: int) -> list:
    """torch.distributed.run command that starts this script on n ranks."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            f"--nproc-per-node={n}", "--master-addr=127.0.0.1", f"--master-port={port}",
            os.path.abspath(__file__)] + list(argv)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=I.WORKLOAD_ORDER, default="qwen3_30b")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override T (smaller cases for profiling; not a bench line)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--l2-flush", choices=["auto", "on", "off"], default="auto",
                    help="write a buffer larger than L2 before every timed step (auto: when "
                         "the step's data is under 4x the L2 size)")
    ap.add_argument("--mode", choices=["forward", "backward"], default="forward",
                    help="backward: time moe_backward instead (one GPU, its own JSON line)")
    ap.add_argument("--check-ranks", action="store_true",
                    help="start the ranks and all-reduce a count vector, time nothing")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.gpus < 1:
        ap.error("--gpus must be at least 1")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # one process per GPU: start this script again under torchrun
        cmd = relaunch_command(sys.argv[1:], args.gpus, free_port())
        raise SystemExit(subprocess.run(cmd).returncode)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but the launcher started {world} ranks")
    if args.check_ranks:
        check_ranks(args, rank, world, local_rank)
        return
    shape = I.WORKLOADS[args.workload]
    if args.tokens is not None:
        shape = shape.replace(T=args.tokens)
    if args.impl == "reference":
        run_reference(args, shape, rank, world)
        return
    if args.mode == "backward":
        if world > 1:
            raise SystemExit("--mode backward runs on one GPU")
        run_backward(args, shape)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, shape, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
