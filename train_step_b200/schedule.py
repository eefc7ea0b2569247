"""Learning-rate schedule of the training recipe: linear warmup, then cosine decay.

The recipe ("AxonLM", Training Recipe table) fixes the peak rate 6e-4, the floor 6e-5
(peak / 10), 715 warmup steps and 19,073 total steps; "AxonLM", Key Features, and
"Genesis", Training Features, name the shape: linear warmup, then cosine decay to the
floor. It does not fix the step indexing; here step s (0-based) of the warmup
uses peak * (s + 1) / warmup, so the first update is not wasted at rate 0, the
cosine runs from the peak at s = warmup to the floor at s = total, and the rate
stays at the floor afterwards.
"""
from __future__ import annotations

import math
from dataclasses import dataclass


@dataclass(frozen=True)
class CosineSchedule:
    max_lr: float = 6e-4
    min_lr: float = 6e-5
    warmup: int = 715
    total: int = 19073

    def __call__(self, step: int) -> float:
        if step < 0:
            raise ValueError("step must be >= 0")
        if step < self.warmup:
            return self.max_lr * (step + 1) / self.warmup
        if step >= self.total:
            return self.min_lr
        frac = (step - self.warmup) / (self.total - self.warmup)
        return self.min_lr + 0.5 * (1.0 + math.cos(math.pi * frac)) * (self.max_lr - self.min_lr)
