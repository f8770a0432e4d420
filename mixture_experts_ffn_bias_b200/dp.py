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
