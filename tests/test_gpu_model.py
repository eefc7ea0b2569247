"""End-to-end parity of the training step (C-ABI handle) against the oracle (GPU).

Tolerances are the ones the target states: fp32 mode, loss relative error <= 1e-5
and per-tensor relative L2 error of gradients and updated parameters <= 1e-4;
bf16 mode, loss relative error <= 2e-3 and per-tensor gradient relative L2 error
<= 2e-2. Relative L2 is ||gpu - ref|| / ||ref||.
"""
import math

import numpy as np
import pytest

import oracle
import train_step_b200 as tsb
from train_step_b200 import synth

pytestmark = pytest.mark.gpu


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b)) if nb == 0 else float(np.linalg.norm(a - b) / nb)


def ocfg(c: tsb.Config) -> oracle.Config:
    return oracle.Config(c.L, c.H, c.C, c.T, c.V, c.tied, c.qkv_bias)


def per_tensor(cfg, a, b, tol, what, skip_key_bias=False):
    """Per-tensor relative L2 check. With skip_key_bias, the key third of each
    qkv bias is left out: its exact gradient is identically zero (adding q.b_k to
    every score of a row leaves the softmax unchanged), so its AdamW update
    g / (|g| + eps) is decided by rounding noise on either side."""
    worst = {}
    for t in oracle.tensors(ocfg(cfg)):
        sl = slice(t.offset, t.offset + t.size)
        x, y = a[sl], b[sl]
        if skip_key_bias and t.name.endswith("qkv_b"):
            keep = np.r_[0:cfg.C, 2 * cfg.C:3 * cfg.C]
            x, y = x[keep], y[keep]
        e = rel_l2(x, y)
        worst[t.name] = e
        assert e <= tol, f"{what} {t.name}: rel L2 {e:.3g} > {tol}"
    return worst


def key_bias_grads(cfg, g):
    out = []
    for t in oracle.tensors(ocfg(cfg)):
        if t.name.endswith("qkv_b"):
            out.append(g[t.offset + cfg.C:t.offset + 2 * cfg.C])
    return np.concatenate(out)


TINY = tsb.Config(L=4, H=4, C=128, T=64, V=65, tied=1, qkv_bias=1, dtype=tsb.FP32, B_max=8)


def test_tensor_table_and_init_match_oracle():
    m = tsb.GPT2(TINY, seed=42)
    names = [t.name for t in oracle.tensors(ocfg(TINY))]
    assert [t[0] for t in m.tensors()] == names
    assert m.num_params == oracle.num_params(ocfg(TINY))
    assert np.array_equal(m.get_params(), oracle.init_params(ocfg(TINY), 42))
    m.close()


def test_tiny_fp32_step_parity():
    """The tiny character-level configuration: one forward+backward and one
    AdamW step (lr 6e-4, wd 0.1, betas 0.9/0.95, clip 1.0)."""
    m = tsb.GPT2(TINY, seed=42)
    oc = ocfg(TINY)
    p0 = m.get_params().astype(np.float64)
    tok, tgt = synth.micro_batch(8, 64, 65, dist="uniform")
    loss = m.forward_backward(tok, tgt)
    rloss, rg = oracle.forward_backward(oc, p0, tok, tgt)
    assert abs(loss - rloss) / abs(rloss) <= 1e-5
    assert abs(loss - math.log(65)) < 0.05
    g = m.get_grads()
    per_tensor(TINY, g, rg, 1e-4, "grad")
    # the key-bias gradient vanishes up to fp32 rounding
    assert np.max(np.abs(key_bias_grads(TINY, g))) <= 1e-6 * np.max(np.abs(rg))
    gn = m.step(6e-4, 0.1, 0.9, 0.95)
    rp, rm, rv, rgn = oracle.adamw_step(oc, p0, rg, np.zeros_like(p0), np.zeros_like(p0), 1, 6e-4, 0.1)
    assert abs(gn - rgn) / rgn <= 1e-4
    per_tensor(TINY, m.get_params(), rp, 1e-4, "param", skip_key_bias=True)
    gm, gv, t = m.get_adam()
    assert t == 1
    per_tensor(TINY, gm, rm, 1e-4, "adam m", skip_key_bias=True)
    per_tensor(TINY, gv, rv, 1e-4, "adam v", skip_key_bias=True)
    # a second step continues from the updated state
    loss2 = m.forward_backward(tok, tgt)
    rloss2, rg2 = oracle.forward_backward(oc, rp, tok, tgt)
    assert abs(loss2 - rloss2) / abs(rloss2) <= 1e-5
    m.step(6e-4, 0.1, 0.9, 0.95)
    rp2, _, _, _ = oracle.adamw_step(oc, rp, rg2, rm, rv, 2, 6e-4, 0.1)
    per_tensor(TINY, m.get_params(), rp2, 1e-4, "param step 2", skip_key_bias=True)
    m.close()


def test_tiny_fp32_accumulation():
    m = tsb.GPT2(TINY, seed=7)
    oc = ocfg(TINY)
    p0 = m.get_params().astype(np.float64)
    grads = []
    for i in range(3):
        tok, tgt = synth.micro_batch(4, 64, 65, index=i, dist="uniform")
        m.forward_backward(tok, tgt, want_loss=False)
        grads.append(oracle.forward_backward(oc, p0, tok, tgt)[1])
    per_tensor(TINY, m.get_grads(), sum(grads) / 3, 1e-4, "accumulated grad")
    m.close()


def _bf16_parity(cfg, B, seed=42, index=0):
    m = tsb.GPT2(cfg, seed=seed)
    oc = ocfg(cfg)
    p0 = m.get_params().astype(np.float64)
    tok, tgt = synth.micro_batch(B, cfg.T, cfg.V, index=index)
    loss = m.forward_backward(tok, tgt)
    rloss, rg = oracle.forward_backward(oc, p0, tok, tgt)
    assert abs(loss - rloss) / abs(rloss) <= 2e-3, (loss, rloss)
    per_tensor(cfg, m.get_grads(), rg, 2e-2, "grad")
    gn = m.step(6e-4, 0.1)
    assert np.isfinite(gn)
    m.close()


def test_bf16_small_tied_parity():
    _bf16_parity(tsb.Config(L=2, H=4, C=256, T=128, V=1000, tied=1, qkv_bias=1, dtype=tsb.BF16, B_max=4), 4)


def test_bf16_small_untied_no_qkv_bias_parity():
    _bf16_parity(tsb.Config(L=2, H=2, C=128, T=200, V=777, tied=0, qkv_bias=0, dtype=tsb.BF16, B_max=3), 3)


def test_bf16_gpt2_width_parity():
    """GPT-2 small width and vocabulary (C=768, H=12, V=50257 -> 50304) with two
    layers and T=256, so that the float64 oracle finishes in seconds."""
    _bf16_parity(tsb.Config(L=2, H=12, C=768, T=256, V=50257, tied=1, qkv_bias=1, dtype=tsb.BF16, B_max=2), 2)


def test_bf16_determinism():
    cfg = tsb.Config(L=2, H=4, C=256, T=128, V=1000, tied=1, qkv_bias=1, dtype=tsb.BF16, B_max=4)
    tok, tgt = synth.micro_batch(4, 128, 1000)
    outs = []
    for _ in range(2):
        m = tsb.GPT2(cfg, seed=3)
        m.forward_backward(tok, tgt)
        outs.append(m.get_grads())
        m.close()
    assert np.array_equal(outs[0], outs[1])


FULL_124M = tsb.Config(L=12, H=12, C=768, T=1024, V=50257, tied=1, qkv_bias=1, dtype=tsb.BF16, B_max=16)


def test_gpt2_124m_full_size():
    """The benchmark's launch configuration (124M, B=16, T=1024, bf16).
    Properties that hold at any size: the batch loss and gradient are the means
    of the per-sequence ones; and the first sequence matches the float64 oracle."""
    m = tsb.GPT2(FULL_124M, seed=42)
    tok, tgt = synth.micro_batch(16, 1024, 50257)
    loss = m.forward_backward(tok, tgt)
    g_batch = m.get_grads()
    assert np.all(np.isfinite(g_batch))
    assert abs(loss - math.log(50257)) < 1.0
    m.zero_grad()
    losses = []
    g_sum = np.zeros_like(g_batch, dtype=np.float64)
    for b in range(16):
        losses.append(m.forward_backward(tok[b:b + 1], tgt[b:b + 1]))
        g_sum += m.get_grads()
        m.zero_grad()
    assert abs(loss - np.mean(losses)) / loss < 1e-3
    per_tensor(FULL_124M, g_batch, g_sum / 16, 2e-2, "batch vs per-sequence grad")
    # sequence 0 against the oracle (float64 forward and backward, T = 1024)
    p0 = m.get_params().astype(np.float64)
    rloss, rg = oracle.forward_backward(ocfg(FULL_124M), p0, tok[:1], tgt[:1])
    assert abs(losses[0] - rloss) / rloss <= 2e-3
    m.forward_backward(tok[:1], tgt[:1], want_loss=False)
    per_tensor(FULL_124M, m.get_grads(), rg, 2e-2, "seq0 grad")
    m.close()


def test_error_paths():
    cfg = tsb.Config(L=1, H=2, C=128, T=32, V=50, tied=1, qkv_bias=1, dtype=tsb.BF16, B_max=2)
    m = tsb.GPT2(cfg, seed=1)
    tok, tgt = synth.micro_batch(2, 32, 50, dist="uniform")
    with pytest.raises(tsb.Gpt2Error) as e:
        m.step(1e-3, 0.1)
    assert e.value.code == -6  # no accumulated gradient
    long_tok, long_tgt = synth.micro_batch(1, 33, 50, dist="uniform")
    with pytest.raises(tsb.Gpt2Error) as e:
        m.forward_backward(long_tok, long_tgt)
    assert e.value.code == -3  # longer than the block size
    big_tok, big_tgt = synth.micro_batch(3, 32, 50, dist="uniform")
    with pytest.raises(tsb.Gpt2Error) as e:
        m.forward_backward(big_tok, big_tgt)
    assert e.value.code == -5  # B > B_max
    bad = tok.copy()
    bad[1, 5] = 50
    with pytest.raises(tsb.Gpt2Error) as e:
        m.forward_backward(bad, tgt)
    assert e.value.code == -4  # token id out of range, caught on the device
    m.zero_grad()
    loss = m.forward_backward(tok, tgt)  # the handle still works
    assert np.isfinite(loss)
    with pytest.raises(tsb.Gpt2Error) as e:
        m.forward_backward(tok[:1], tgt[:1])
    assert e.value.code == -5  # B changes inside one accumulation
    m.close()
    with pytest.raises(tsb.Gpt2Error) as e:
        tsb.GPT2(tsb.Config(L=1, H=3, C=128, T=8, V=10, dtype=tsb.BF16))
    assert e.value.code == -1
