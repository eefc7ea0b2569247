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


def shard_bounds(n: int, world: int, rank: int) -> tuple[int, int]:
    """Storage range [lo, hi) of rank `rank`'s shard: W equal pieces, each a multiple of 64
    floats (the library's storage length is a multiple of 4096)."""
    if n % (64 * world):
        raise ValueError(f"storage length {n} does not split into {world} shards of 64-float multiples")
    shard = n // world
    return rank * shard, (rank + 1) * shard


def reduce_scatter_mean_(tensor, lo: int, hi: int, group=None) -> None:
    """tensor[lo:hi] <- the average over the ranks of their tensor[lo:hi] (this rank's
    shard of an equal split). NCCL reduces in place into the shard; gloo, which has no
    reduce-scatter, all-reduces the whole tensor (the same values in the shard)."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    if world == 1:
        return
    if dist.get_backend(group) == "nccl":
        out = torch.empty_like(tensor[lo:hi])
        dist.reduce_scatter_tensor(out, tensor, op=dist.ReduceOp.AVG, group=group)
        tensor[lo:hi].copy_(out)
    else:
        dist.all_reduce(tensor, op=dist.ReduceOp.SUM, group=group)
        tensor.div_(world)


def all_gather_shards_(tensor, lo: int, hi: int, group=None) -> None:
    """Every rank's shard tensor[lo_r:hi_r] into every rank's tensor (in place)."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    if world == 1:
        return
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(tensor, tensor[lo:hi].clone(), group=group)
    else:
        parts = [torch.empty_like(tensor[lo:hi]) for _ in range(world)]
        dist.all_gather(parts, tensor[lo:hi].contiguous(), group=group)
        torch.cat(parts, out=tensor)


def zero1_step(model, lr: float, wd: float, beta1: float = 0.9, beta2: float = 0.95, group=None) -> None:
    """One optimizer step with the optimizer sharded over the ranks (ZeRO stage 1):
    reduce-scatter of the accumulated gradients, the global norm from every shard's sum
    of squares, AdamW on this rank's shard of parameters and moments, all-gather of the
    updated parameter shards, refresh of the bf16 weight shadow, gradients zeroed. Gives
    the update of an all-reduce followed by the full step (same clip, same AdamW). All
    work runs on torch's current stream, which must be the model's stream."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    g = model.grad_tensor()
    lo, hi = shard_bounds(g.numel(), world, rank)
    reduce_scatter_mean_(g, lo, hi, group)
    ss = torch.zeros(1, dtype=torch.float64, device=g.device)
    model.grad_sumsq(lo, hi, ss)
    if world > 1:
        dist.all_reduce(ss, op=dist.ReduceOp.SUM, group=group)
    model.step_range(lr, wd, beta1, beta2, lo, hi, ss)
    all_gather_shards_(model.param_tensor(), lo, hi, group)
    model.refresh_shadow()
    model.zero_grad()


class BucketedAllReduce:
    """Average of the accumulated gradients over the ranks, one bucket at a time (bucket l
    holds layer l's tensors, bucket L the embeddings, final LayerNorm and untied head),
    each bucket's all-reduce starting on a stream of its own as soon as the backward pass
    of the last micro-batch has finished that bucket (gpt2_set_grad_events), so the
    exchange overlaps the rest of that backward pass. Reverse layer order, as the
    backward pass produces them.

        ex = BucketedAllReduce(model)
        for i, (tok, tgt) in enumerate(micro_batches):
            if i == len(micro_batches) - 1:
                ex.arm()
            model.forward_backward(tok, tgt, want_loss=False)
        ex.run()        # enqueues the exchange and orders the current stream after it
        model.step(...)

    The model must run on torch's current stream. Without CUDA (a CPU process group and
    a CPU gradient tensor) run() reduces the buckets in the same order, synchronously.
    """

    def __init__(self, model, group=None, ranges=None):
        import torch
        from . import bucket_ranges
        self.model, self.group = model, group
        self.L = model.cfg.L
        self.ranges = ranges if ranges is not None else bucket_ranges(model.cfg)
        self.order = list(range(self.L - 1, -1, -1)) + [self.L]
        self.cuda = torch.cuda.is_available() and model.grad_tensor().is_cuda
        self.events = []
        if self.cuda:
            self.stream = torch.cuda.Stream()
            self.events = [torch.cuda.Event() for _ in range(self.L + 1)]
            for e in self.events:  # creates the CUDA events (completed at once)
                e.record()
        self.armed = False

    def arm(self) -> None:
        """Before the last micro-batch's forward_backward."""
        if self.cuda:
            self.model.set_grad_events(self.events)
        self.armed = True

    def run(self) -> None:
        """After the last micro-batch's forward_backward has returned: the all-reduces,
        each waiting for its bucket; then the current stream waits for all of them."""
        import torch
        import torch.distributed as dist
        if not self.armed:
            raise RuntimeError("arm() before the last micro-batch")
        self.armed = False
        g = self.model.grad_tensor()
        world = dist.get_world_size(self.group) if dist.is_available() and dist.is_initialized() else 1
        if not self.cuda:
            if world > 1:
                for b in self.order:
                    for off, n in self.ranges[b]:
                        allreduce_mean_(g[off:off + n], self.group)
            return
        with torch.cuda.stream(self.stream):
            for b in self.order:
                self.stream.wait_event(self.events[b])
                if world > 1:
                    for off, n in self.ranges[b]:
                        allreduce_mean_(g[off:off + n], self.group)
        torch.cuda.current_stream().wait_stream(self.stream)
