"""Training driver on the GPU: the loss falls under the warmup + cosine schedule, and a
checkpoint taken between steps resumes to bit-identical parameters (every kernel of the
step is deterministic).
"""
import numpy as np
import pytest
import torch

import train_step_b200 as tsb
from train_step_b200 import synth
from train_step_b200.schedule import CosineSchedule
from train_step_b200.trainer import Trainer

pytestmark = pytest.mark.gpu

SMALL = tsb.Config(L=2, H=4, C=256, T=128, V=1000, tied=1, qkv_bias=1, dtype=tsb.BF16, B_max=4)


def _batches(n, index0=0):
    out = []
    for i in range(n):
        tok, tgt = synth.micro_batch(4, SMALL.T, SMALL.V, index=index0 + i)
        out.append((torch.from_numpy(tok).cuda(), torch.from_numpy(tgt).cuda()))
    return out


def test_loss_decreases_under_schedule():
    model = tsb.GPT2(SMALL, seed=3)
    tr = Trainer(model, CosineSchedule(max_lr=2e-3, min_lr=2e-4, warmup=5, total=40))
    train = _batches(2)
    held = _batches(2, index0=100)
    first = tr.train_step(train)
    eval0 = tr.eval_loss(held)
    for _ in range(39):
        last = tr.train_step(train)
    assert tr.step == 40
    assert last["lr"] == pytest.approx(CosineSchedule(2e-3, 2e-4, 5, 40)(39))
    assert last["loss"] < first["loss"] - 1.0       # the repeated batches are being fitted
    assert tr.eval_loss(held) < eval0               # and held-out batches improve too
    model.close()


def test_checkpoint_resume_is_bit_identical(tmp_path):
    sched = CosineSchedule(max_lr=1e-3, min_lr=1e-4, warmup=2, total=10)
    batches = [_batches(2, index0=10 * s) for s in range(5)]
    a = tsb.GPT2(SMALL, seed=5)
    ta = Trainer(a, sched)
    for s in range(3):
        ta.train_step(batches[s])
    path = str(tmp_path / "ck.npz")
    ta.save(path)
    for s in range(3, 5):
        ta.train_step(batches[s])
    pa, (ma, va, t_a) = a.get_params(), a.get_adam()

    b = tsb.GPT2(SMALL, seed=99)  # different initialisation, overwritten by the checkpoint
    tb = Trainer(b, sched)
    tb.load(path)
    assert tb.step == 3
    for s in range(3, 5):
        tb.train_step(batches[s])
    pb, (mb, vb, t_b) = b.get_params(), b.get_adam()
    assert t_a == t_b == 5
    assert np.array_equal(pa, pb) and np.array_equal(ma, mb) and np.array_equal(va, vb)
    a.close()
    b.close()
