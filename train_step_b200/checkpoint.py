"""Checkpoint and resume: parameters, Adam moments and step count in one .npz file.

A checkpoint is taken between optimizer steps (no gradients are pending): it holds the
fp32 parameters and the Adam moments m, v in canonical order (12 bytes per parameter,
1.49 GB at 124M), the Adam step count t, the caller's step counter and the model
configuration, which `load` checks against the target model ("AxonLM", Key Features:
checkpoint resume; "gpt/docs/LLM.md", Memory Footprint: about 1.49 GB with optimizer states).
"""
from __future__ import annotations

import json
import os
from dataclasses import asdict

import numpy as np


def save(model, path: str, step: int = 0, extra: dict | None = None) -> None:
    """Write the checkpoint to `path` (exactly that name) through a temporary file in the
    same directory and an atomic rename, so that an interrupted save never leaves a
    truncated file under `path`."""
    params = model.get_params()
    m, v, t = model.get_adam()
    tmp = f"{path}.tmp.{os.getpid()}"
    with open(tmp, "wb") as f:
        np.savez(f, params=params, adam_m=m, adam_v=v, adam_t=np.int64(t), step=np.int64(step),
                 config=json.dumps(asdict(model.cfg), sort_keys=True), extra=json.dumps(extra or {}))
    os.replace(tmp, path)


def load(model, path: str) -> tuple[int, dict]:
    """Restore `model` from `path`; returns (step, extra)."""
    with np.load(path) as d:
        cfg = json.loads(str(d["config"]))
        if cfg != json.loads(json.dumps(asdict(model.cfg), sort_keys=True)):
            raise ValueError(f"checkpoint configuration {cfg} does not match the model's {asdict(model.cfg)}")
        model.set_params(d["params"])
        model.set_adam(d["adam_m"], d["adam_v"], int(d["adam_t"]))
        return int(d["step"]), json.loads(str(d["extra"]))
