"""World-size-2 gloo test of the data-parallel exchange (CPU, no GPU).

Each rank routes its own token shard (the oracle stands in for the GPU
forward, which cannot run here), sums counts with the same helper the
benchmark uses, and applies the bias update.  Both ranks must end with the
same bias, equal to the single-process update from the whole batch; without
the all-reduce the replicas drift apart (the failure the page-2 README warns
about)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from mixture_experts_ffn_bias_b200 import inputs as I
from mixture_experts_ffn_bias_b200.dp import allreduce_counts
from oracle import moe_oracle as O

SHAPE = I.WORKLOADS["skew"].replace(T=1024, d_model=128, d_ff=128, d_ff_shared=128)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _local_counts(rank, world, host):
    lo, hi = rank * SHAPE.T // world, (rank + 1) * SHAPE.T // world
    r = O.router(host["x"][lo:hi], host["w_router"], SHAPE.top_k, SHAPE.gate, True,
                 host["sel_bias"], host["logit_offset"])
    return O.dispatch(r.topk_idx, SHAPE.n_experts).counts


def _worker(rank, world, port, q, do_allreduce):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        host = I.make_inputs(SHAPE)
        c = torch.from_numpy(_local_counts(rank, world, host).astype(np.int32))
        if do_allreduce:
            allreduce_counts(c)
        bias = O.bias_update(c.numpy(), host["sel_bias"])
        q.put((rank, c.numpy().tolist(), bias.tolist()))
    finally:
        dist.destroy_process_group()


def _run(world, do_allreduce):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q, do_allreduce))
             for r in range(world)]
    for p in procs:
        p.start()
    res = dict((r, (c, b)) for r, c, b in (q.get(timeout=120) for _ in procs))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return res


def test_counts_allreduce_keeps_replicas_identical():
    res = _run(2, True)
    host = I.make_inputs(SHAPE)
    full = _local_counts(0, 1, host)
    ref_bias = O.bias_update(full, host["sel_bias"])
    for r in (0, 1):
        assert res[r][0] == full.tolist()
        np.testing.assert_array_equal(np.array(res[r][1], np.float32), ref_bias)


def test_without_allreduce_replicas_drift():
    res = _run(2, False)
    assert res[0][1] != res[1][1]


def test_single_process_is_a_noop():
    c = torch.arange(5, dtype=torch.int32)
    assert allreduce_counts(c).tolist() == [0, 1, 2, 3, 4]


def _grad_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from mixture_experts_ffn_bias_b200.dp import allreduce_grads
        host = I.make_inputs(GSHAPE)
        dout = np.random.default_rng(3).standard_normal((GSHAPE.T, GSHAPE.d_model))
        lo, hi = rank * GSHAPE.T // world, (rank + 1) * GSHAPE.T // world
        shard = dict(host)
        shard["x"] = host["x"][lo:hi]
        g = O.moe_backward(shard, GSHAPE.top_k, GSHAPE.gate, True, dout[lo:hi])
        grads = {k: torch.from_numpy(g[k]) for k in ("dw_router", "dw1", "dw3", "dw2", "dws1",
                                                     "dws3", "dws2")}
        allreduce_grads(grads)
        q.put((rank, {k: v.numpy() for k, v in grads.items()}))
    finally:
        dist.destroy_process_group()


GSHAPE = I.WORKLOADS["skew"].replace(T=96, d_model=16, n_experts=8, d_ff=8, d_ff_shared=8,
                                     top_k=2)


def test_weight_gradients_summed_over_shards_equal_full_batch():
    """Data-parallel backward: each rank differentiates its own token shard
    (the oracle stands in for moe_backward, which needs a GPU); the
    all-reduced weight gradients equal the gradients of the whole batch,
    since every weight gradient is a sum over tokens."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_grad_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    host = I.make_inputs(GSHAPE)
    dout = np.random.default_rng(3).standard_normal((GSHAPE.T, GSHAPE.d_model))
    full = O.moe_backward(host, GSHAPE.top_k, GSHAPE.gate, True, dout)
    for r in (0, 1):
        for k, v in res[r].items():
            np.testing.assert_allclose(v, full[k], rtol=1e-9, atol=1e-12, err_msg=k)


def test_bench_launches_one_rank_per_gpu():
    """bench.py --gpus 2 without a torchrun environment starts itself again on
    two ranks; --check-ranks makes them all-reduce a count vector (gloo here)
    and rank 0 reports the world size it saw."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2",
                        "--check-ranks"], capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(s) for s in r.stdout.splitlines() if s.startswith("{")]
    assert len(lines) == 1
    assert lines[0]["world_size"] == 2 and lines[0]["counts_allreduce_ok"]


def test_bench_refuses_a_world_size_that_differs_from_gpus():
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2",
                        "--check-ranks"], capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode != 0 and "launcher started 1 ranks" in r.stderr
