"""Data-parallel replicas of the layer: the one exchange on the path.

Every rank runs the whole layer on its own tokens.  Before the selection-bias
update the per-expert counts are summed over the ranks, so every replica
applies the same update ("moe-200m-qwen3-100b" README, "Per-layer numerics"
and the caller-side snippet after step_bias_update: all-reduce the counts
before the bias update, otherwise the per-rank biases drift apart and DDP's
buffer broadcast discards half of the signal).
"""
from __future__ import annotations


def allreduce_counts(counts, group=None):
    """Sum int32 per-expert counts over the process group, in place (NCCL on
    GPUs, gloo on CPU).  A no-op when torch.distributed is not initialised or
    the group has one rank."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(counts, op=dist.ReduceOp.SUM, group=group)
    return counts


def allreduce_grads(grads, keys=("dw_router", "dw1", "dw3", "dw2", "dws1", "dws3", "dws2"),
                    group=None, average=False):
    """Sum (or average) the weight gradients of a moe_backward call over the
    process group, in place, as one flat buffer per dtype (one collective per
    dtype instead of one per tensor; 16-bit gradients are summed in fp32).  dx stays per rank: it
    belongs to the rank's own tokens.  The weight gradients of a layer are
    sums over tokens, so the sum over token shards equals the gradient of
    the whole batch; average=True gives the mean that data-parallel
    optimisers apply.  A no-op without an initialised multi-rank group."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1):
        return grads
    world = dist.get_world_size(group)
    names = [k for k in keys if grads.get(k) is not None]
    by_dtype = {}
    for k in names:
        by_dtype.setdefault(grads[k].dtype, []).append(k)
    for dtype, ks in by_dtype.items():
        # 16-bit gradients are summed in fp32; wider ones in their own dtype
        acc = torch.float32 if dtype in (torch.bfloat16, torch.float16) else dtype
        flat = torch.cat([grads[k].reshape(-1).to(acc) for k in ks])
        dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
        if average:
            flat /= world
        off = 0
        for k in ks:
            n = grads[k].numel()
            grads[k].copy_(flat[off:off + n].view_as(grads[k]).to(dtype))
            off += n
    return grads
