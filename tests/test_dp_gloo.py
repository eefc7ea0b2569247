"""Data-parallel host logic on CPU with two gloo ranks: sharding micro-batches by
rank and averaging gradients gives the same update as one process accumulating
all the micro-batches (float64 oracle as the compute)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CFG = dict(L=2, H=2, C=32, T=16, V=29, tied=1, qkv_bias=1)
ACCUM = 2


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, out_dir):
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import oracle
    from train_step_b200 import dp, synth
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    oc = oracle.Config(**CFG)
    p = oracle.init_params(oc, 5).astype(np.float64)
    g = np.zeros_like(p)
    for idx in dp.micro_batch_indices(rank, world, ACCUM):
        tok, tgt = synth.micro_batch(2, CFG["T"], CFG["V"], index=idx, dist="uniform")
        g += oracle.forward_backward(oc, p, tok, tgt)[1]
    t = torch.from_numpy(g)
    dp.allreduce_mean_(t)
    G = t.numpy() / ACCUM
    p1, _, _, gn = oracle.adamw_step(oc, p, G, np.zeros_like(p), np.zeros_like(p), 1, 6e-4, 0.1)
    np.save(os.path.join(out_dir, f"p{rank}.npy"), p1)
    dist.barrier()
    dist.destroy_process_group()


def test_micro_batch_indices_partition():
    seen = []
    for r in range(4):
        seen += __import__("train_step_b200.dp", fromlist=["x"]).micro_batch_indices(r, 4, 3, step=1)
    assert sorted(seen) == list(range(12, 24))


def test_two_rank_gloo_matches_single_process(tmp_path):
    import oracle
    from train_step_b200 import dp, synth
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    p_r = [np.load(tmp_path / f"p{r}.npy") for r in range(world)]
    assert np.array_equal(p_r[0], p_r[1])  # every rank applies the same update
    oc = oracle.Config(**CFG)
    p = oracle.init_params(oc, 5).astype(np.float64)
    g = np.zeros_like(p)
    idx = [i for r in range(world) for i in dp.micro_batch_indices(r, world, ACCUM)]
    for i in idx:
        tok, tgt = synth.micro_batch(2, CFG["T"], CFG["V"], index=i, dist="uniform")
        g += oracle.forward_backward(oc, p, tok, tgt)[1]
    p1, _, _, _ = oracle.adamw_step(oc, p, g / len(idx), np.zeros_like(p), np.zeros_like(p), 1, 6e-4, 0.1)
    assert np.max(np.abs(p_r[0] - p1)) < 1e-15


class _OracleModel:
    """The Trainer's model interface on the float64 oracle (CPU): gradients accumulate in a
    torch buffer that the data-parallel all-reduce averages, as on the GPU handle."""

    def __init__(self, seed):
        import oracle
        self.oc = oracle.Config(**CFG)
        self.p = oracle.init_params(self.oc, seed).astype(np.float64)
        self.m = np.zeros_like(self.p)
        self.v = np.zeros_like(self.p)
        self.t = 0
        self.k = 0
        self.gbuf = torch.zeros(self.p.size, dtype=torch.float64)

    def forward_backward(self, tok, tgt):
        import oracle
        loss, g = oracle.forward_backward(self.oc, self.p, tok, tgt)
        self.gbuf += torch.from_numpy(g)
        self.k += 1
        return loss

    def forward(self, tok, tgt):
        import oracle
        return oracle.forward(self.oc, self.p, tok, tgt)

    def step(self, lr, wd, b1, b2):
        import oracle
        self.t += 1
        G = self.gbuf.numpy() / self.k
        self.p, self.m, self.v, gn = oracle.adamw_step(self.oc, self.p, G, self.m, self.v, self.t, lr, wd, b1, b2)
        self.gbuf.zero_()
        self.k = 0
        return gn


def _trainer_rank(rank, world, port, out_dir):
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from train_step_b200 import dp, synth
    from train_step_b200.schedule import CosineSchedule
    from train_step_b200.trainer import Trainer
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    model = _OracleModel(9)
    tr = Trainer(model, CosineSchedule(1e-3, 1e-4, 1, 4), allreduce=lambda: dp.allreduce_mean_(model.gbuf))
    lrs = []
    for step in range(3):
        mbs = [synth.micro_batch(2, CFG["T"], CFG["V"], index=i, dist="uniform")
               for i in dp.micro_batch_indices(rank, world, ACCUM, step=step)]
        lrs.append(tr.train_step(mbs)["lr"])
    np.save(os.path.join(out_dir, f"tp{rank}.npy"), model.p)
    np.save(os.path.join(out_dir, f"lr{rank}.npy"), np.array(lrs))
    dist.barrier()
    dist.destroy_process_group()


def test_trainer_two_rank_gloo_matches_single_process(tmp_path):
    """Three optimizer steps of the training driver on two gloo ranks (each its own
    micro-batches, gradients averaged before AdamW) equal one process accumulating all of
    them, and the learning rates follow the oracle's schedule."""
    import oracle
    from train_step_b200 import dp, synth
    from train_step_b200.schedule import CosineSchedule
    from train_step_b200.trainer import Trainer
    world = 2
    mp.start_processes(_trainer_rank, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn")
    p_r = [np.load(tmp_path / f"tp{r}.npy") for r in range(world)]
    assert np.array_equal(p_r[0], p_r[1])
    model = _OracleModel(9)
    tr = Trainer(model, CosineSchedule(1e-3, 1e-4, 1, 4))
    for step in range(3):
        idx = [i for r in range(world) for i in dp.micro_batch_indices(r, world, ACCUM, step=step)]
        tr.train_step([synth.micro_batch(2, CFG["T"], CFG["V"], index=i, dist="uniform") for i in idx])
    assert np.max(np.abs(p_r[0] - model.p)) < 1e-12
    lrs = np.load(tmp_path / "lr0.npy")
    assert np.allclose(lrs, [oracle.lr_schedule(s, 1e-3, 1e-4, 1, 4) for s in range(3)], rtol=0, atol=1e-18)
