"""Training driver around the C-ABI model: gradient accumulation, optional data-parallel
gradient averaging, the warmup + cosine learning-rate schedule, AdamW, evaluation loss
and checkpoints ("AxonLM", Training Recipe and Key Features: cosine schedule with warmup,
checkpoint resume; "GPT From Scratch", Key decisions: warmup plus cosine decay, clipping at
1.0, gradient accumulation).
"""
from __future__ import annotations

from typing import Callable, Iterable

from . import checkpoint
from .schedule import CosineSchedule


def _sync_torch_stream() -> None:
    try:
        import torch
    except ImportError:
        return
    if torch.cuda.is_available() and torch.cuda.is_initialized():
        torch.cuda.current_stream().synchronize()


class Trainer:
    """`exchange` (e.g. dp.BucketedAllReduce; the model on torch's current stream) averages
    the gradients over data-parallel ranks while the last micro-batch's backward pass
    runs, ordered by streams alone; `allreduce` (a callable run after the backward pass,
    on torch's current stream) is the plain form, followed by a host synchronisation."""

    def __init__(self, model, schedule: Callable[[int], float] | None = None, weight_decay: float = 0.1,
                 beta1: float = 0.9, beta2: float = 0.95, allreduce: Callable[[], None] | None = None,
                 exchange=None):
        self.model = model
        self.schedule = schedule or CosineSchedule()
        self.weight_decay = weight_decay
        self.beta1 = beta1
        self.beta2 = beta2
        self.allreduce = allreduce
        self.exchange = exchange
        self.step = 0

    def train_step(self, micro_batches: Iterable) -> dict:
        """One optimizer step over the (tokens, targets) micro-batches: returns the mean
        micro-batch loss, the pre-clip gradient norm and the learning rate used."""
        if self.exchange is not None:
            mbs = list(micro_batches)
            losses = []
            for i, (tok, tgt) in enumerate(mbs):
                if i == len(mbs) - 1:
                    self.exchange.arm()
                    self.model.forward_backward(tok, tgt, want_loss=False)
                    self.exchange.run()  # enqueued before the host waits for the loss
                    losses.append(self.model.read_loss())
                else:
                    losses.append(self.model.forward_backward(tok, tgt))
            lr = self.schedule(self.step)
            gnorm = self.model.step(lr, self.weight_decay, self.beta1, self.beta2)
            self.step += 1
            return {"loss": sum(losses) / len(losses), "grad_norm": gnorm, "lr": lr, "step": self.step}
        losses = [self.model.forward_backward(tok, tgt) for tok, tgt in micro_batches]
        if self.allreduce is not None:
            # the gradients are complete (each forward_backward returned its loss); the
            # collective runs on torch's current stream, which the optimizer step on the
            # model's own stream must not overtake
            self.allreduce()
            _sync_torch_stream()
        lr = self.schedule(self.step)
        gnorm = self.model.step(lr, self.weight_decay, self.beta1, self.beta2)
        self.step += 1
        return {"loss": sum(losses) / len(losses), "grad_norm": gnorm, "lr": lr, "step": self.step}

    def eval_loss(self, batches: Iterable) -> float:
        losses = [self.model.forward(tok, tgt) for tok, tgt in batches]
        return sum(losses) / len(losses)

    def save(self, path: str) -> None:
        checkpoint.save(self.model, path, step=self.step)

    def load(self, path: str) -> None:
        self.step, _ = checkpoint.load(self.model, path)
