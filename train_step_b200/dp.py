"""Data-parallel plumbing around the single-GPU step ("AxonLM", Quick Start:
torchrun with DistributedDataParallel over 8 GPUs).

Each rank trains on its own micro-batches; the one exchange per optimizer step
is an average of the accumulated gradients across ranks (NCCL over NVLink on
GPUs, gloo on CPU), after which every rank applies the same AdamW update to
identical parameters.
"""
from __future__ import annotations


def micro_batch_indices(rank: int, world: int, accum: int, step: int = 0) -> list[int]:
    """Global indices of the micro-batches rank `rank` processes in `step`:
    rank r of W takes [step*W*accum + r*accum, ... + accum)."""
    base = step * world * accum + rank * accum
    return list(range(base, base + accum))


def allreduce_mean_(tensor, group=None) -> None:
    """In-place average of `tensor` over the ranks of `group`."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    if world == 1:
        return
    if dist.get_backend(group) == "nccl":
        dist.all_reduce(tensor, op=dist.ReduceOp.AVG, group=group)
    else:
        dist.all_reduce(tensor, op=dist.ReduceOp.SUM, group=group)
        tensor.div_(world)
