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


class _ShardedFlatModel:
    """Float64 CPU stand-in for the library's sharded-step interface (ZeRO stage 1), to
    test the host logic of dp.zero1_step: flat storage in canonical order padded to a
    multiple of 4096, gradients accumulated as a sum over k micro-batches, and the
    documented range update (norm sqrt(sumsq) / k, clip 1/(norm + 1e-6) capped at 1,
    AdamW with decay on the >= 2-D tensors)."""

    def __init__(self, seed):
        import oracle
        self.oc = oracle.Config(**CFG)
        p0 = oracle.init_params(self.oc, seed).astype(np.float64)
        self.P = p0.size
        n = (self.P + 4095) // 4096 * 4096
        self.p = np.zeros(n)
        self.p[:self.P] = p0
        self.m = np.zeros(n)
        self.v = np.zeros(n)
        self.decay = np.zeros(n, dtype=bool)
        for t in oracle.tensors(self.oc):
            self.decay[t.offset:t.offset + t.size] = t.decay
        self.g = torch.zeros(n, dtype=torch.float64)
        self.k = 0
        self.t = 0

    def forward_backward(self, tok, tgt):
        import oracle
        loss, g = oracle.forward_backward(self.oc, self.p[:self.P], tok, tgt)
        self.g[:self.P] += torch.from_numpy(g)
        self.k += 1
        return loss

    def grad_tensor(self):
        return self.g

    def param_tensor(self):
        return torch.from_numpy(self.p)

    def grad_sumsq(self, lo, hi, out):
        out[0] = float((self.g[lo:hi] ** 2).sum())

    def step_range(self, lr, wd, b1, b2, lo, hi, sumsq):
        self.t += 1
        norm = np.sqrt(float(sumsq[0])) / self.k
        coef = min(1.0, 1.0 / (norm + 1e-6))
        gg = self.g[lo:hi].numpy() * (coef / self.k)
        p, m, v, d = self.p[lo:hi], self.m[lo:hi], self.v[lo:hi], self.decay[lo:hi]
        p[d] *= 1.0 - lr * wd
        m[:] = b1 * m + (1.0 - b1) * gg
        v[:] = b2 * v + (1.0 - b2) * gg * gg
        p -= lr * (m / (1.0 - b1 ** self.t)) / (np.sqrt(v / (1.0 - b2 ** self.t)) + 1e-8)
        self.k = 0

    def refresh_shadow(self):
        pass

    def zero_grad(self):
        self.g.zero_()
        self.k = 0


def _zero1_rank(rank, world, port, out_dir):
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from train_step_b200 import dp, synth
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    model = _ShardedFlatModel(11)
    for step in range(2):
        for i in dp.micro_batch_indices(rank, world, ACCUM, step=step):
            model.forward_backward(*synth.micro_batch(2, CFG["T"], CFG["V"], index=i, dist="uniform"))
        dp.zero1_step(model, 6e-4, 0.1)
    np.save(os.path.join(out_dir, f"z{rank}.npy"), model.p[:model.P])
    np.save(os.path.join(out_dir, f"zm{rank}.npy"), model.m)
    dist.barrier()
    dist.destroy_process_group()


def test_shard_bounds_partition():
    from train_step_b200 import dp
    n = 4096 * 3
    for world in (1, 2, 4, 8, 64):
        cuts = [dp.shard_bounds(n, world, r) for r in range(world)]
        assert cuts[0][0] == 0 and cuts[-1][1] == n
        assert all(a[1] == b[0] for a, b in zip(cuts, cuts[1:]))
        assert all(lo % 64 == 0 and (hi - lo) == n // world for lo, hi in cuts)
    with pytest.raises(ValueError):
        dp.shard_bounds(4096 + 64, 2, 0)


def test_zero1_two_rank_gloo_matches_single_process(tmp_path):
    """Two optimizer steps with the optimizer sharded over two gloo ranks (reduce-scatter,
    the norm from the shards' sums of squares, AdamW on each rank's half, all-gather)
    give the parameters of one process taking the full step on all micro-batches, and
    each rank's moments are non-zero only on its own half."""
    import oracle
    from train_step_b200 import dp, synth
    world = 2
    mp.start_processes(_zero1_rank, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    p_r = [np.load(tmp_path / f"z{r}.npy") for r in range(world)]
    assert np.array_equal(p_r[0], p_r[1])
    oc = oracle.Config(**CFG)
    p = oracle.init_params(oc, 11).astype(np.float64)
    m = np.zeros_like(p)
    v = np.zeros_like(p)
    for step in range(2):
        idx = [i for r in range(world) for i in dp.micro_batch_indices(r, world, ACCUM, step=step)]
        g = np.zeros_like(p)
        for i in idx:
            g += oracle.forward_backward(oc, p, *synth.micro_batch(2, CFG["T"], CFG["V"], index=i, dist="uniform"))[1]
        p, m, v, _ = oracle.adamw_step(oc, p, g / len(idx), m, v, step + 1, 6e-4, 0.1)
    assert np.max(np.abs(p_r[0] - p)) < 1e-12
    n = np.load(tmp_path / "zm0.npy").size
    for r in range(world):
        mr = np.load(tmp_path / f"zm{r}.npy")
        lo, hi = dp.shard_bounds(n, world, r)
        assert np.all(mr[:lo] == 0) and np.all(mr[hi:] == 0) and np.any(mr[lo:hi] != 0)


def _tsb_cfg(cfg):
    import train_step_b200 as tsb
    return tsb.Config(L=cfg["L"], H=cfg["H"], C=cfg["C"], T=cfg["T"], V=cfg["V"], tied=cfg["tied"],
                      qkv_bias=cfg["qkv_bias"])


@pytest.mark.parametrize("cfg", [dict(CFG, C=64), dict(L=12, H=12, C=768, T=1024, V=50257, tied=1, qkv_bias=1),
                                 dict(L=12, H=12, C=768, T=1024, V=50257, tied=0, qkv_bias=0),
                                 dict(L=48, H=25, C=1600, T=1024, V=50257, tied=1, qkv_bias=1)])
def test_gradient_buckets_cover_the_storage(cfg):
    """The library's storage layout (a host-only query): each tensor lies inside one range
    of its own bucket, the buckets' ranges are disjoint, and bucket l holds exactly layer
    l's tensors."""
    import train_step_b200 as tsb
    c = _tsb_cfg(cfg)
    layout, n_store = tsb.storage_layout(c)
    ranges = tsb.bucket_ranges(c)
    assert len(ranges) == c.L + 1
    for name, off, n, b in layout:
        assert b == (int(name[1:name.index(".")]) if name[0] == "h" and name[1].isdigit() else c.L)
        assert sum(1 for o, m in ranges[b] if o <= off and off + n <= o + m) == 1, name
    flat = sorted(r for rs in ranges for r in rs)
    assert all(a[0] + a[1] <= b[0] for a, b in zip(flat, flat[1:]))
    assert flat[-1][0] + flat[-1][1] <= n_store
    covered = sum(n for _, _, n, _ in layout)
    assert covered <= sum(m for _, m in flat) <= covered + 64 * len(layout)


class _StorageOracleModel:
    """The float64 oracle behind the library's gradient storage layout (CPU): gradients
    accumulate into a flat buffer laid out as the library lays out its own (offsets and
    padding from gpt2_storage_layout), which the bucketed exchange averages range by
    range; the step gathers them back into canonical order for the oracle's AdamW."""

    def __init__(self, seed):
        import oracle
        import train_step_b200 as tsb
        self.cfg = _tsb_cfg(dict(CFG, C=64))
        self.oc = oracle.Config(**dict(CFG, C=64))
        self.p = oracle.init_params(self.oc, seed).astype(np.float64)
        self.m = np.zeros_like(self.p)
        self.v = np.zeros_like(self.p)
        self.t = 0
        self.k = 0
        layout, n_store = tsb.storage_layout(self.cfg)
        self.map = []  # (canonical offset, storage offset, logical length)
        for (name, off, n, _), t in zip(layout, oracle.tensors(self.oc)):
            assert name.split(".")[-1] == t.name.split(".")[-1] and t.size <= n
            self.map.append((t.offset, off, t.size))
        self.g = torch.zeros(n_store, dtype=torch.float64)
        self.last = None

    def grad_tensor(self):
        return self.g

    def set_grad_events(self, events):
        pass

    def forward_backward(self, tok, tgt, want_loss=True):
        import oracle
        loss, g = oracle.forward_backward(self.oc, self.p, tok, tgt)
        for co, so, n in self.map:
            self.g[so:so + n] += torch.from_numpy(g[co:co + n])
        self.k += 1
        self.last = loss
        return loss if want_loss else None

    def read_loss(self):
        return self.last

    def step(self, lr, wd, b1, b2):
        import oracle
        G = np.zeros_like(self.p)
        for co, so, n in self.map:
            G[co:co + n] = self.g[so:so + n].numpy()
        self.t += 1
        self.p, self.m, self.v, gn = oracle.adamw_step(self.oc, self.p, G / self.k, self.m, self.v, self.t, lr, wd,
                                                       b1, b2)
        self.g.zero_()
        self.k = 0
        return gn


def _bucketed_rank(rank, world, port, out_dir):
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from train_step_b200 import dp, synth
    from train_step_b200.schedule import CosineSchedule
    from train_step_b200.trainer import Trainer
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    model = _StorageOracleModel(13)
    tr = Trainer(model, CosineSchedule(1e-3, 1e-4, 1, 4), exchange=dp.BucketedAllReduce(model))
    losses = []
    for step in range(3):
        mbs = [synth.micro_batch(2, CFG["T"], CFG["V"], index=i, dist="uniform")
               for i in dp.micro_batch_indices(rank, world, ACCUM, step=step)]
        losses.append(tr.train_step(mbs)["loss"])
    np.save(os.path.join(out_dir, f"bp{rank}.npy"), model.p)
    np.save(os.path.join(out_dir, f"bl{rank}.npy"), np.array(losses))
    dist.barrier()
    dist.destroy_process_group()


def test_bucketed_exchange_two_rank_gloo_matches_single_process(tmp_path):
    """Three steps of the training driver with the bucketed exchange (gradients averaged
    bucket by bucket, reverse layer order, over the library's storage layout) on two gloo
    ranks equal one process accumulating every micro-batch; the reported loss is the mean
    of the rank's own micro-batch losses."""
    from train_step_b200 import dp, synth
    from train_step_b200.schedule import CosineSchedule
    from train_step_b200.trainer import Trainer
    world = 2
    mp.start_processes(_bucketed_rank, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn")
    p_r = [np.load(tmp_path / f"bp{r}.npy") for r in range(world)]
    assert np.array_equal(p_r[0], p_r[1])
    model = _StorageOracleModel(13)
    tr = Trainer(model, CosineSchedule(1e-3, 1e-4, 1, 4))
    for step in range(3):
        idx = [i for r in range(world) for i in dp.micro_batch_indices(r, world, ACCUM, step=step)]
        tr.train_step([synth.micro_batch(2, CFG["T"], CFG["V"], index=i, dist="uniform") for i in idx])
    assert np.max(np.abs(p_r[0] - model.p)) < 1e-12
    l0 = np.load(tmp_path / "bl0.npy")
    assert np.all(np.isfinite(l0)) and l0.shape == (3,)
