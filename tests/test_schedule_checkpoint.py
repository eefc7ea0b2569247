"""Learning-rate schedule and checkpoint file format (CPU).

The oracle's schedule is pinned to values the recipe fixes ("AxonLM", Training Recipe
table: peak 6e-4, minimum 6e-5, 715 warmup steps, 19,073 total) and to closed-form
properties of a linear warmup and a half-cosine; the library's schedule must agree with it.
"""
import numpy as np
import pytest

import oracle
from train_step_b200 import checkpoint
from train_step_b200.schedule import CosineSchedule


def test_oracle_schedule_pins():
    lr = oracle.lr_schedule
    assert lr(0) == pytest.approx(6e-4 / 715, rel=1e-15)           # first warmup step
    assert lr(714) == pytest.approx(6e-4, rel=1e-15)               # end of warmup reaches the peak
    assert lr(715) == pytest.approx(6e-4, rel=1e-15)               # cosine starts at the peak
    assert lr(19073) == pytest.approx(6e-5, rel=1e-15)             # and ends at peak / 10
    assert lr(10**6) == pytest.approx(6e-5, rel=1e-15)             # then stays there
    mid = (715 + 19073) // 2                                       # half way: the mean of the two
    assert lr(mid) == pytest.approx((6e-4 + 6e-5) / 2, rel=1e-12)
    for x in (1, 100, 4589, 9000):                                 # the half-cosine is point-symmetric
        assert lr(715 + x) + lr(19073 - x) == pytest.approx(6e-4 + 6e-5, rel=1e-12)
    warm = [lr(s) for s in range(715)]
    assert np.allclose(np.diff(warm), 6e-4 / 715, rtol=1e-9)        # linear warmup
    decay = [lr(s) for s in range(715, 19074, 97)]
    assert all(a >= b for a, b in zip(decay, decay[1:]))          # monotone decay


def test_library_schedule_matches_oracle():
    sched = CosineSchedule()
    for s in list(range(0, 800)) + list(range(800, 20000, 37)):
        assert sched(s) == pytest.approx(oracle.lr_schedule(s), rel=1e-12, abs=0.0)
    short = CosineSchedule(max_lr=1e-3, min_lr=1e-4, warmup=5, total=30)
    for s in range(40):
        assert short(s) == pytest.approx(oracle.lr_schedule(s, 1e-3, 1e-4, 5, 30), rel=1e-12)
    with pytest.raises(ValueError):
        sched(-1)


class _FakeModel:
    """Stands in for tsb.GPT2 on the host: the checkpoint module only uses these calls."""

    def __init__(self, cfg, n, seed):
        rng = np.random.default_rng(seed)
        self.cfg = cfg
        self.p = rng.standard_normal(n).astype(np.float32)
        self.m = rng.standard_normal(n).astype(np.float32)
        self.v = rng.random(n).astype(np.float32)
        self.t = int(rng.integers(1, 100))

    def get_params(self):
        return self.p.copy()

    def set_params(self, p):
        self.p = np.array(p, np.float32)

    def get_adam(self):
        return self.m.copy(), self.v.copy(), self.t

    def set_adam(self, m, v, t):
        self.m, self.v, self.t = np.array(m, np.float32), np.array(v, np.float32), int(t)


def test_checkpoint_round_trip(tmp_path):
    from train_step_b200 import Config
    cfg = Config(L=1, H=2, C=8, T=4, V=11)
    a = _FakeModel(cfg, 1000, 1)
    path = str(tmp_path / "ck.npz")
    checkpoint.save(a, path, step=17, extra={"note": "x"})
    b = _FakeModel(cfg, 1000, 2)
    step, extra = checkpoint.load(b, path)
    assert step == 17 and extra == {"note": "x"}
    assert np.array_equal(a.p, b.p) and np.array_equal(a.m, b.m) and np.array_equal(a.v, b.v) and a.t == b.t
    c = _FakeModel(Config(L=2, H=2, C=8, T=4, V=11), 1000, 3)
    with pytest.raises(ValueError):
        checkpoint.load(c, path)


def test_checkpoint_payload_and_atomic_name(tmp_path):
    # 12 bytes per parameter (fp32 p, m, v): 1.49 GB at 124,439,808 parameters, the figure
    # "gpt/docs/LLM.md" (Memory Footprint) gives for a checkpoint with optimizer state
    from train_step_b200 import Config
    cfg = Config(L=1, H=2, C=8, T=4, V=11)
    a = _FakeModel(cfg, 5000, 4)
    path = str(tmp_path / "ckpt")  # no extension: the file is written under exactly this name
    checkpoint.save(a, path, step=3)
    assert sorted(p.name for p in tmp_path.iterdir()) == ["ckpt"]
    with np.load(path) as d:
        payload = sum(d[k].nbytes for k in ("params", "adam_m", "adam_v"))
        assert all(d[k].dtype == np.float32 for k in ("params", "adam_m", "adam_v"))
    assert payload == 12 * 5000
    assert abs(12 * 124_439_808 / 1e9 - 1.49) < 0.01
