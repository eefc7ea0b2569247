"""Parity of the exact code paths the full-size training step takes (GPU).

The end-to-end tests elsewhere run small models whose launches differ from the
benchmark's: one partial head chunk, no split-K, a single micro-batch. This file
checks against the float64 oracle what only the full-size step exercises:
  * the GEMM launches of the 124M step at their real shapes, through the library's
    own choice of tile, 2-CTA pairing and split-K (sampled output rows);
  * a bf16 model whose B*T spans two head chunks, accumulated over two micro-batches,
    then its optimizer step (updated master weights, moments, norm) and a forward
    that reads the refreshed bf16 weight shadow;
  * the forward-only call (evaluation loss) in both precisions;
  * the GPT-2 medium and XL widths (C = 1024 / H = 16 and C = 1600 / H = 25, where
    3C = 4800 is not a multiple of the 256-wide tile);
  * the out-of-memory and bounded-wait error codes, made without any GPU fault.
Tolerances: fp32 GEMM accumulation 1e-5 relative L2 (as the per-op tests); the
model-level bars of the target (bf16: loss 2e-3, gradients 2e-2; fp32: loss 1e-5,
updated parameters and moments 1e-4).
"""
import numpy as np
import pytest
import torch

import oracle
import train_step_b200 as tsb
from train_step_b200 import synth

pytestmark = pytest.mark.gpu

DEV = "cuda"


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b)) if nb == 0 else float(np.linalg.norm(a - b) / nb)


def g64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def randn(shape, seed, dtype=torch.bfloat16, scale=1.0):
    gen = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=gen, dtype=torch.float32) * scale).to(dtype).to(DEV)


def ocfg(c):
    return oracle.Config(c.L, c.H, c.C, c.T, c.V, c.tied, c.qkv_bias)


def per_tensor(cfg, a, b, tol, what):
    for t in oracle.tensors(ocfg(cfg)):
        sl = slice(t.offset, t.offset + t.size)
        e = rel_l2(a[sl], b[sl])
        assert e <= tol, f"{what} {t.name}: rel L2 {e:.3g} > {tol}"


# ---------------------------------------------------------------------------
# GEMM launches of the 124M step (B = 16, T = 1024: N = 16,384 rows; C = 768,
# F = 3072, Vp = 50,304; head chunks of 4096 rows)
# ---------------------------------------------------------------------------
# (name, M, N, K, a_mn, b_mn): the operand majors the step passes
STEP_GEMMS = [
    ("fc dW (split-K)", 3072, 768, 16384, True, True),   # dW_fc = du^T h2
    ("head dX", 4096, 768, 50304, False, True),          # dxf = dlogits W
    ("head dW", 50304, 768, 4096, True, True),           # dW_head = dlogits^T xf
    ("qkv forward", 16384, 2304, 768, False, False),     # qkv = h1 W^T
]


@pytest.mark.parametrize("name,M,N,K,a_mn,b_mn", STEP_GEMMS, ids=[g[0] for g in STEP_GEMMS])
def test_step_gemm_at_full_size(name, M, N, K, a_mn, b_mn):
    """One launch with the library's own tile, pair and split-K choice (the timing entry
    point with ksplit 0, bn 0, pair -1, one warm-up launch and one timed launch, both
    storing the same result), checked on sampled output rows spread over every tile row
    and the ragged tail."""
    A_st = randn((K, M) if a_mn else (M, K), 31)
    B_st = randn((K, N) if b_mn else (N, K), 32, scale=0.05)
    out = torch.full((M, N), float("nan"), dtype=torch.float32, device=DEV)
    tsb.gemm_bench(A_st, B_st, out, M=M, N=N, K=K, lda=M if a_mn else K, ldb=N if b_mn else K, ldo=N, a_mn=a_mn,
                   b_mn=b_mn, epilogue=tsb.EPI_F32, ksplit=0, bn=0, pair=-1, iters=1)
    torch.cuda.synchronize()
    rng = np.random.default_rng(M + N + K)
    rows = np.unique(np.concatenate([rng.choice(M, 120, replace=False), np.arange(M - 8, M),
                                     np.arange(0, M, max(1, M // 64))]))
    A_rows = (A_st[:, rows].t() if a_mn else A_st[rows]).contiguous()
    B_log = (B_st.t() if b_mn else B_st).contiguous()
    ref = oracle.linear_fwd(g64(A_rows), g64(B_log))
    got = g64(out[torch.from_numpy(rows).to(DEV)])
    assert np.all(np.isfinite(got))
    # fp32 accumulation of K exact bf16 products: the rounding error of a length-K sum grows
    # like sqrt(K) units of 2^-24 (random-walk bound; a factor 4 covers the tensor core's
    # accumulation order, measured 1.9e-5 at K = 50,304). The per-op bar of 1e-5 stays the
    # floor for short sums.
    tol = max(1e-5, 4.0 * (K ** 0.5) * 2.0 ** -24)
    assert rel_l2(got, ref) < tol, (name, rel_l2(got, ref), tol)


# ---------------------------------------------------------------------------
# A bf16 model over two head chunks, two micro-batches, then the optimizer step
# ---------------------------------------------------------------------------
TWO_CHUNKS = tsb.Config(L=1, H=2, C=128, T=1024, V=4099, tied=1, qkv_bias=1, dtype=tsb.BF16, B_max=5)


def test_bf16_two_head_chunks_accumulation_and_step():
    cfg = TWO_CHUNKS
    assert 5 * 1024 > 4096  # B*T spans a full 4096-row chunk and a ragged second one
    oc = ocfg(cfg)
    m = tsb.GPT2(cfg, seed=11)
    p0 = m.get_params().astype(np.float64)
    ref_g = np.zeros_like(p0)
    for i in range(2):
        tok, tgt = synth.micro_batch(5, cfg.T, cfg.V, index=20 + i)
        loss = m.forward_backward(tok, tgt)
        rloss, rg = oracle.forward_backward(oc, p0, tok, tgt)
        assert abs(loss - rloss) / abs(rloss) <= 2e-3, (i, loss, rloss)
        ref_g += rg
    g = m.get_grads()  # (1/k) sum over the two micro-batches
    per_tensor(cfg, g, ref_g / 2, 2e-2, "accumulated grad")
    # the optimizer step of the bf16 handle on its own gradients, against the oracle's
    # AdamW (clip, decay on the 2-D prefix, bias correction) applied to the same gradients
    lr, wd = 1e-2, 0.1
    gn = m.step(lr, wd, 0.9, 0.95)
    rp, rm, rv, rgn = oracle.adamw_step(oc, p0, g.astype(np.float64), np.zeros_like(p0), np.zeros_like(p0), 1, lr, wd)
    assert abs(gn - rgn) / rgn <= 1e-5
    p1 = m.get_params()
    gm, gv, t = m.get_adam()
    assert t == 1
    per_tensor(cfg, p1, rp, 1e-4, "param")
    per_tensor(cfg, gm, rm, 1e-4, "adam m")
    per_tensor(cfg, gv, rv, 1e-4, "adam v")
    # the GEMMs now read the refreshed bf16 shadow: the forward loss is the oracle's at the
    # updated master weights (a stale shadow would give the pre-step loss, far outside 2e-3)
    tok, tgt = synth.micro_batch(5, cfg.T, cfg.V, index=20)
    before = oracle.forward(oc, p0, tok, tgt)
    after_ref = oracle.forward(oc, p1.astype(np.float64), tok, tgt)
    assert abs(after_ref - before) / abs(before) > 2e-2
    after = m.forward(tok, tgt)
    assert abs(after - after_ref) / abs(after_ref) <= 2e-3, (after, after_ref, before)
    m.close()


# ---------------------------------------------------------------------------
# The forward-only call (evaluation loss)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("cfg,dist,tol", [
    (tsb.Config(L=4, H=4, C=128, T=64, V=65, tied=1, qkv_bias=1, dtype=tsb.FP32, B_max=8), "uniform", 1e-5),
    (tsb.Config(L=2, H=4, C=256, T=256, V=3000, tied=0, qkv_bias=1, dtype=tsb.BF16, B_max=3), "zipf", 2e-3),
], ids=["fp32-tiny", "bf16-untied"])
def test_forward_only_loss(cfg, dist, tol):
    m = tsb.GPT2(cfg, seed=5)
    p = m.get_params().astype(np.float64)
    for i in range(2):
        tok, tgt = synth.micro_batch(cfg.B_max, cfg.T, cfg.V, index=40 + i, dist=dist)
        loss = m.forward(tok, tgt)
        rloss = oracle.forward(ocfg(cfg), p, tok, tgt)
        assert abs(loss - rloss) / abs(rloss) <= tol, (i, loss, rloss)
    with pytest.raises(tsb.Gpt2Error) as e:
        m.step(1e-3, 0.1)  # forward only: nothing accumulated
    assert e.value.code == -6
    m.close()


# ---------------------------------------------------------------------------
# GPT-2 medium and XL widths
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("C,H", [(1024, 16), (1600, 25)], ids=["355M-width", "1558M-width"])
def test_bf16_medium_and_xl_widths(C, H):
    cfg = tsb.Config(L=1, H=H, C=C, T=256, V=3001, tied=1, qkv_bias=1, dtype=tsb.BF16, B_max=2)
    m = tsb.GPT2(cfg, seed=42)
    p0 = m.get_params().astype(np.float64)
    tok, tgt = synth.micro_batch(2, cfg.T, cfg.V, index=3)
    loss = m.forward_backward(tok, tgt)
    rloss, rg = oracle.forward_backward(ocfg(cfg), p0, tok, tgt)
    assert abs(loss - rloss) / abs(rloss) <= 2e-3, (loss, rloss)
    per_tensor(cfg, m.get_grads(), rg, 2e-2, "grad")
    m.close()


# ---------------------------------------------------------------------------
# Error codes made without any GPU fault
# ---------------------------------------------------------------------------
def test_out_of_memory_is_reported_and_the_device_stays_usable():
    # ~2.4e11 parameters: the first state allocation (fp32 parameters, ~966 GB) fails
    huge = tsb.Config(L=300, H=128, C=8192, T=64, V=1000, tied=1, qkv_bias=1, dtype=tsb.BF16, B_max=1)
    with pytest.raises(tsb.Gpt2Error) as e:
        tsb.GPT2(huge, seed=1)
    assert e.value.code == -2
    cfg = tsb.Config(L=1, H=2, C=128, T=32, V=50, tied=1, qkv_bias=1, dtype=tsb.BF16, B_max=2)
    m = tsb.GPT2(cfg, seed=1)
    tok, tgt = synth.micro_batch(2, 32, 50, dist="uniform")
    assert np.isfinite(m.forward_backward(tok, tgt))
    m.close()


def test_bounded_wait_reports_timeout_and_the_context_survives():
    tsb.bounded_wait_check(True, 1_000_000)  # completed barrier: no error
    with pytest.raises(tsb.Gpt2Error) as e:
        tsb.bounded_wait_check(False, 0)  # nobody arrives: the wait gives up at once
    assert e.value.code == -8
    with pytest.raises(tsb.Gpt2Error) as e:
        tsb.bounded_wait_check(False, 200_000)  # gives up after 0.2 ms
    assert e.value.code == -8
    tsb.bounded_wait_check(True, 0)
    x = torch.ones(1024, device=DEV)
    assert float(x.sum()) == 1024.0


# ---------------------------------------------------------------------------
# The sharded optimizer step (ZeRO stage 1) of the data-parallel path
# ---------------------------------------------------------------------------
def test_sharded_step_equals_the_full_step():
    """Two 'ranks' emulated by two handles with identical gradients: each updates one half
    of the storage with the global squared norm summed from both halves; the halves put
    together (the all-gather) give the full gpt2_step's parameters and norm, and the
    refreshed bf16 shadow gives the same forward loss."""
    cfg = tsb.Config(L=2, H=2, C=128, T=64, V=500, tied=1, qkv_bias=1, dtype=tsb.BF16, B_max=2)
    models = [tsb.GPT2(cfg, seed=3) for _ in range(3)]
    batches = [synth.micro_batch(2, 64, 500, index=i) for i in range(2)]
    for mdl in models:
        for tok, tgt in batches:
            mdl.forward_backward(tok, tgt, want_loss=False)
    gn = models[0].step(6e-4, 0.1, 0.9, 0.95)
    _, n = models[1].grad_buffer()
    assert n % 4096 == 0
    half = n // 2
    s = [torch.zeros(1, dtype=torch.float64, device=DEV) for _ in range(2)]
    models[1].grad_sumsq(0, half, s[0])
    models[2].grad_sumsq(half, n, s[1])
    tot = s[0] + s[1]
    torch.cuda.synchronize()
    gn1 = models[1].step_range(6e-4, 0.1, 0.9, 0.95, 0, half, tot, want_norm=True)
    gn2 = models[2].step_range(6e-4, 0.1, 0.9, 0.95, half, n, tot, want_norm=True)
    assert abs(gn1 - gn) <= 1e-6 * gn and gn1 == gn2
    models[1].param_tensor()[half:].copy_(models[2].param_tensor()[half:])
    torch.cuda.synchronize()
    models[1].refresh_shadow()
    models[1].zero_grad()
    p_full, p_shard = models[0].get_params(), models[1].get_params()
    assert rel_l2(p_shard, p_full) <= 1e-6
    tok, tgt = synth.micro_batch(2, 64, 500, index=7)
    l0, l1 = models[0].forward(tok, tgt), models[1].forward(tok, tgt)
    assert abs(l1 - l0) <= 1e-5 * abs(l0)
    for mdl in models:
        mdl.close()


# ---------------------------------------------------------------------------
# Gradient-bucket events of the overlapped data-parallel exchange
# ---------------------------------------------------------------------------
def test_grad_bucket_events_and_the_overlapped_exchange():
    """gpt2_set_grad_events: the next backward pass records one event per gradient bucket,
    in the order L-1, ..., 0, L (device timestamps), leaves the gradients bit-identical to
    a run without events and the loss readable later (gpt2_read_loss); the training
    driver with the bucketed exchange (one process: the exchange only waits on the events)
    takes the same steps as without it."""
    from train_step_b200 import dp
    from train_step_b200.schedule import CosineSchedule
    from train_step_b200.trainer import Trainer
    cfg = tsb.Config(L=3, H=2, C=128, T=128, V=1000, tied=1, qkv_bias=1, dtype=tsb.BF16, B_max=2)
    stream = torch.cuda.current_stream().cuda_stream
    a = tsb.GPT2(cfg, seed=3, stream=stream)
    b = tsb.GPT2(cfg, seed=3, stream=stream)
    tok, tgt = synth.micro_batch(2, cfg.T, cfg.V, index=7)
    events = [torch.cuda.Event(enable_timing=True) for _ in range(cfg.L + 1)]
    for e in events:
        e.record()
    torch.cuda.synchronize()
    a.set_grad_events(events)
    a.forward_backward(tok, tgt, want_loss=False)
    la = a.read_loss()
    lb = b.forward_backward(tok, tgt)
    torch.cuda.synchronize()
    assert la == lb
    order = list(range(cfg.L - 1, -1, -1)) + [cfg.L]
    for x, y in zip(order, order[1:]):
        assert events[x].elapsed_time(events[y]) >= 0.0, (x, y)
    assert np.array_equal(a.get_grads(), b.get_grads())
    # one-shot: a later backward pass does not record the events again (the marker recorded
    # between the two calls stays after every bucket event)
    marker = torch.cuda.Event(enable_timing=True)
    marker.record()
    a.forward_backward(tok, tgt, want_loss=False)
    torch.cuda.synchronize()
    assert all(e.elapsed_time(marker) >= 0.0 for e in events)
    # armed, then a forward-only call: the events wait for the next backward pass
    a.set_grad_events(events)
    a.forward(tok, tgt)
    marker.record()
    a.forward_backward(tok, tgt, want_loss=False)
    torch.cuda.synchronize()
    assert all(marker.elapsed_time(e) >= 0.0 for e in events)
    with pytest.raises(tsb.Gpt2Error) as e:
        a.set_grad_events(events[:2])
    assert e.value.code == -1
    a.zero_grad()
    b.zero_grad()
    sched = CosineSchedule(1e-3, 1e-4, 1, 4)
    ta = Trainer(a, sched, exchange=dp.BucketedAllReduce(a))
    tb = Trainer(b, sched)
    for step in range(2):
        mbs = [synth.micro_batch(2, cfg.T, cfg.V, index=10 + 2 * step + i) for i in range(2)]
        ra, rb = ta.train_step(mbs), tb.train_step(mbs)
        assert ra["loss"] == rb["loss"] and ra["grad_norm"] == rb["grad_norm"]
    assert np.array_equal(a.get_params(), b.get_params())
    a.close()
    b.close()


# ---------------------------------------------------------------------------
# Overlap does not change a bit: side-stream reductions and programmatic dependent launches
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("C,H", [(256, 4), (1600, 25)], ids=["C256", "C1600"])
def test_overlapped_and_in_order_runs_are_bitwise_equal(C, H):
    """The bf16 step normally overlaps gradient reductions on a second stream and launches its
    kernels as programmatic dependents; with per-kernel profiling on, everything runs in order
    on one stream with ordinary launches. Every reduction has a fixed order, so the two must
    agree bit for bit: losses, accumulated gradients and the parameters after a step. A missing
    wait in either mechanism would show up here as a difference."""
    cfg = tsb.Config(L=2, H=H, C=C, T=256, V=3001, tied=1, qkv_bias=1, dtype=tsb.BF16, B_max=4)
    batches = [synth.micro_batch(4, cfg.T, cfg.V, index=60 + i) for i in range(3)]
    out = []
    for in_order in (False, True):
        m = tsb.GPT2(cfg, seed=17)
        if in_order:
            m.profile(True)
        losses = [m.forward_backward(tok, tgt) for tok, tgt in batches]
        g = m.get_grads()
        gn = m.step(1e-3, 0.1, 0.9, 0.95)
        out.append((losses, g, gn, m.get_params()))
        m.close()
    (la, ga, na, pa), (lb, gb, nb, pb) = out
    assert la == lb
    assert np.array_equal(ga, gb)
    assert na == nb
    assert np.array_equal(pa, pb)
