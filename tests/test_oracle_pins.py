"""Pins of the float64 oracle to facts outside itself (CPU only).

Each test checks the oracle against something the pages print, a closed form,
an invariant, finite differences, or a float64 library routine, so that a
dropped term, a wrong sign or index, or a transposed operand fails at least one.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from train_step_b200 import synth

TINY = oracle.Config(L=4, H=4, C=128, T=64, V=65, tied=1, qkv_bias=1)
MICRO = oracle.Config(L=2, H=2, C=8, T=5, V=11, tied=1, qkv_bias=1)
MICRO_UNTIED = oracle.Config(L=2, H=2, C=8, T=5, V=11, tied=0, qkv_bias=1)


def rand_params(cfg, seed, scale=1.0):
    """Init-spec weights with LN gains/biases and linear biases perturbed, so
    that every parameter has a nonzero gradient path."""
    p = oracle.init_params(cfg, seed).astype(np.float64)
    rng = np.random.default_rng(seed)
    for t in oracle.tensors(cfg):
        sl = slice(t.offset, t.offset + t.size)
        if len(t.shape) == 1:
            p[sl] += 0.1 * rng.standard_normal(t.size)
        else:
            p[sl] *= scale
    return p


def batch(cfg, B, index=0, dist="uniform"):
    return synth.micro_batch(B, cfg.T, cfg.V, index=index, dist=dist)


# --------------------------------------------------------------------------
# Numbers printed on the pages
# --------------------------------------------------------------------------
def test_param_count_124m_tied(golden):
    cfg = oracle.Config(12, 12, 768, 1024, golden["vocab_logical"], tied=1, qkv_bias=1)
    assert oracle.num_params(cfg) == golden["param_count_gpt2_124m_tied_v50257"]


def test_param_count_untied_163m(golden):
    # The untied figure matches a model without QKV bias; with the bias it would
    # be 12 * 2304 larger.
    cfg = oracle.Config(12, 12, 768, 1024, golden["vocab_logical"], tied=0, qkv_bias=0)
    assert oracle.num_params(cfg) == golden["param_count_untied_163m"]
    cfg_b = oracle.Config(12, 12, 768, 1024, golden["vocab_logical"], tied=0, qkv_bias=1)
    assert oracle.num_params(cfg_b) == golden["param_count_untied_163m"] + 12 * 3 * 768


def test_state_bytes_match_checkpoint_size(golden):
    # fp32 params + Adam m + v = 12 bytes/param ~ 1.49 GB for the 124M model.
    n = oracle.num_params(oracle.Config(12, 12, 768, 1024, 50257))
    assert abs(12 * n / 1e9 - golden["checkpoint_gb_with_optimizer"]) < 0.01


def test_tiny_init_loss_near_ln_vocab(golden):
    p = oracle.init_params(TINY, 42)
    tok, tgt = batch(TINY, 8)
    loss = oracle.forward(TINY, p, tok, tgt)
    assert abs(loss - math.log(golden["tiny_vocab"])) < 0.05


def test_init_statistics():
    cfg = oracle.Config(L=4, H=4, C=128, T=64, V=65)
    p = oracle.init_params(cfg, 7)
    for t in oracle.tensors(cfg):
        x = p[t.offset:t.offset + t.size].astype(np.float64)
        if t.name.endswith(("ln1_g", "ln2_g", "lnf_g")):
            assert np.all(x == 1.0)
        elif len(t.shape) == 1:
            assert np.all(x == 0.0)
        else:
            sigma = 0.02 / math.sqrt(2 * cfg.L) if t.name.endswith(("ao_w", "pj_w")) else 0.02
            assert abs(x.mean()) < 5 * sigma / math.sqrt(x.size)
            assert abs(x.std() / sigma - 1) < 6 / math.sqrt(2 * x.size) + 0.01


# --------------------------------------------------------------------------
# Invariants the pages name
# --------------------------------------------------------------------------
def test_causality_exact():
    p = rand_params(TINY, 3)
    tok, tgt = batch(TINY, 2)
    _, z0 = oracle.forward(TINY, p, tok, tgt, want_logits=True)
    t = 20
    tok2 = tok.copy()
    tok2[:, t + 1:] = (tok2[:, t + 1:] + 17) % TINY.V
    _, z1 = oracle.forward(TINY, p, tok2, tgt, want_logits=True)
    z0 = z0.reshape(2, TINY.T, -1)
    z1 = z1.reshape(2, TINY.T, -1)
    assert np.array_equal(z0[:, :t + 1], z1[:, :t + 1])
    assert not np.array_equal(z0[:, t + 1:], z1[:, t + 1:])


def test_two_attention_formulations_agree():
    rng = np.random.default_rng(0)
    B, T, NH, hd = 2, 37, 3, 16
    qkv = rng.standard_normal((B * T, 3 * NH * hd))
    o0, l0 = oracle.attention_fwd(qkv, B, T, NH, hd, mode=0)
    o1, l1 = oracle.attention_fwd(qkv, B, T, NH, hd, mode=1)
    assert np.max(np.abs(o0 - o1)) <= 1e-10
    assert np.max(np.abs(l0 - l1)) <= 1e-10
    # the whole model with either formulation
    p = rand_params(TINY, 4)
    tok, tgt = batch(TINY, 2)
    a = oracle.forward(TINY, p, tok, tgt, attn_mode=0)
    b = oracle.forward(TINY, p, tok, tgt, attn_mode=1)
    assert abs(a - b) <= 1e-10


def test_attention_first_row_is_v0():
    rng = np.random.default_rng(1)
    B, T, NH, hd = 1, 9, 2, 8
    qkv = rng.standard_normal((B * T, 3 * NH * hd))
    C = NH * hd
    for mode in (0, 1):
        o, lse = oracle.attention_fwd(qkv, B, T, NH, hd, mode=mode)
        assert np.array_equal(o[0], qkv[0, 2 * C:3 * C])
        # lse of row 0 is the single scaled score
        for h in range(NH):
            q = qkv[0, h * hd:(h + 1) * hd]
            k = qkv[0, C + h * hd:C + (h + 1) * hd]
            assert abs(lse[0, h, 0] - q @ k / math.sqrt(hd)) < 1e-14


def test_attention_matches_torch_sdpa():
    rng = np.random.default_rng(2)
    B, T, NH, hd = 2, 33, 4, 16
    C = NH * hd
    qkv = rng.standard_normal((B * T, 3 * C))
    o, _ = oracle.attention_fwd(qkv, B, T, NH, hd, mode=0)
    t = torch.from_numpy(qkv).view(B, T, 3, NH, hd)
    q, k, v = (t[:, :, i].transpose(1, 2) for i in range(3))
    ref = F.scaled_dot_product_attention(q, k, v, is_causal=True).transpose(1, 2).reshape(B * T, C)
    assert np.max(np.abs(o - ref.numpy())) < 1e-12


def test_attention_bwd_matches_autograd():
    rng = np.random.default_rng(3)
    B, T, NH, hd = 2, 19, 2, 8
    C = NH * hd
    qkv = rng.standard_normal((B * T, 3 * C))
    dout = rng.standard_normal((B * T, C))
    d = oracle.attention_bwd(qkv, dout, B, T, NH, hd)
    t = torch.from_numpy(qkv).requires_grad_(True)
    v = t.view(B, T, 3, NH, hd)
    q, k, vv = (v[:, :, i].transpose(1, 2) for i in range(3))
    o = F.scaled_dot_product_attention(q, k, vv, is_causal=True).transpose(1, 2).reshape(B * T, C)
    o.backward(torch.from_numpy(dout))
    assert np.max(np.abs(d - t.grad.numpy())) < 1e-12


def test_layernorm_invariants_and_library():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((50, 96)) * 3 + 1.5
    g = np.ones(96)
    b = np.zeros(96)
    y, mean, rstd = oracle.layernorm_fwd(x, g, b)
    assert np.max(np.abs(y.mean(1))) < 1e-13
    # biased variance with eps 1e-5: var(y) = var / (var + eps)
    var = x.var(1)
    assert np.max(np.abs(y.var(1) - var / (var + 1e-5))) < 1e-12
    g = rng.standard_normal(96)
    b = rng.standard_normal(96)
    y, mean, rstd = oracle.layernorm_fwd(x, g, b)
    ref = F.layer_norm(torch.from_numpy(x), (96,), torch.from_numpy(g), torch.from_numpy(b), eps=1e-5)
    assert np.max(np.abs(y - ref.numpy())) < 1e-12
    dy = rng.standard_normal(x.shape)
    dx, dg, db = oracle.layernorm_bwd(dy, x, g, mean, rstd)
    # sum over the row of dx vanishes when g is constant
    dx1, _, _ = oracle.layernorm_bwd(dy, x, np.full(96, 0.7), mean, rstd)
    assert np.max(np.abs(dx1.sum(1))) < 1e-12
    xt = torch.from_numpy(x).requires_grad_(True)
    gt = torch.from_numpy(g).requires_grad_(True)
    bt = torch.from_numpy(b).requires_grad_(True)
    F.layer_norm(xt, (96,), gt, bt, eps=1e-5).backward(torch.from_numpy(dy))
    assert np.max(np.abs(dx - xt.grad.numpy())) < 1e-11
    assert np.max(np.abs(dg - gt.grad.numpy())) < 1e-11
    assert np.max(np.abs(db - bt.grad.numpy())) < 1e-11


def test_gelu_tanh_matches_library_and_limits():
    u = np.linspace(-8, 8, 1001)
    a = oracle.gelu_fwd(u)
    ref = F.gelu(torch.from_numpy(u), approximate="tanh").numpy()
    assert np.max(np.abs(a - ref)) < 1e-14
    assert oracle.gelu_fwd(np.array([0.0]))[0] == 0.0
    # within 1e-3 of the exact erf form everywhere
    exact = 0.5 * u * (1 + np.vectorize(math.erf)(u / math.sqrt(2)))
    assert np.max(np.abs(a - exact)) < 1e-3
    du = oracle.gelu_bwd(u, np.ones_like(u))
    ut = torch.from_numpy(u).requires_grad_(True)
    F.gelu(ut, approximate="tanh").sum().backward()
    assert np.max(np.abs(du - ut.grad.numpy())) < 1e-13


def test_cross_entropy_library_and_grad_rows_sum_to_zero():
    rng = np.random.default_rng(5)
    N, V, ld = 40, 65, 128
    z = rng.standard_normal((N, ld)) * 2
    z[:, V:] = 1e3  # padding columns must be ignored
    tgt = rng.integers(0, V, N).astype(np.int32)
    tot, rl, dl = oracle.cross_entropy(z, V, tgt, scale=1.0 / N)
    ref = F.cross_entropy(torch.from_numpy(z[:, :V]), torch.from_numpy(tgt).long(), reduction="none").numpy()
    assert np.max(np.abs(rl - ref)) < 1e-12
    assert abs(tot - ref.sum()) < 1e-10
    assert np.max(np.abs(dl.sum(1))) < 1e-15
    assert np.all(dl[:, V:] == 0)
    zt = torch.from_numpy(z[:, :V].copy()).requires_grad_(True)
    F.cross_entropy(zt, torch.from_numpy(tgt).long()).backward()
    assert np.max(np.abs(dl[:, :V] - zt.grad.numpy())) < 1e-15


def test_token_buckets_are_a_stable_counting_sort():
    tok, _ = synth.micro_batch(4, 256, 50257, dist="zipf")
    counts, offsets, pos = oracle.token_buckets(tok, 50257)
    flat = tok.ravel()
    assert np.array_equal(counts, np.bincount(flat, minlength=50257))
    assert np.array_equal(offsets, np.concatenate([[0], np.cumsum(counts)[:-1]]))
    assert np.array_equal(pos, np.argsort(flat, kind="stable"))


def test_embedding_fwd_is_a_gather_plus_position_rows():
    # "gpt/docs/LLM.md", Embedding Layer: token embedding plus learned position
    # embedding; position t is the index within its own sequence. B = 3 and a
    # position table longer than T make any other position index (n / B, n without
    # the modulus, a transposed [T, B] order) pick different rows.
    rng = np.random.default_rng(5)
    B, T, Tmax, C, V = 3, 7, 11, 6, 23
    tok, _ = synth.micro_batch(B, T, V, dist="uniform")
    wte = rng.standard_normal((V, C))
    wpe = rng.standard_normal((Tmax, C))
    x0 = oracle.embedding_fwd(tok, wte, wpe)
    ref = (wte[tok] + wpe[np.arange(T)][None, :, :]).reshape(B * T, C)
    assert np.array_equal(x0, ref)


def test_model_embedding_step_is_the_exported_one():
    # The model's forward adds position row t to position t of EVERY sequence of the
    # batch: perturbing wpe row t leaves every earlier position of every sequence
    # unchanged (causality) and changes position t of every sequence.
    cfg = oracle.Config(L=1, H=2, C=8, T=6, V=13, tied=1, qkv_bias=1)
    p = rand_params(cfg, 9)
    tok, tgt = synth.micro_batch(3, cfg.T, cfg.V, dist="uniform")
    _, z0 = oracle.forward(cfg, p, tok, tgt, want_logits=True)
    wpe = next(t for t in oracle.tensors(cfg) if t.name == "wpe")
    t = 4
    p2 = p.copy()
    p2[wpe.offset + t * cfg.C:wpe.offset + (t + 1) * cfg.C] += 0.5
    _, z1 = oracle.forward(cfg, p2, tok, tgt, want_logits=True)
    d = np.abs(z1 - z0).reshape(3, cfg.T, cfg.V).max(axis=2)
    # causal: positions before t unchanged in every sequence; position t changed in every sequence
    assert np.all(d[:, :t] == 0.0)
    assert np.all(d[:, t] > 0.0)


def test_embedding_bwd_matches_scatter_add():
    rng = np.random.default_rng(6)
    tok, _ = synth.micro_batch(3, 20, 97, dist="zipf")
    dx0 = rng.standard_normal((60, 12))
    dwte, dwpe = oracle.embedding_bwd(tok, dx0, 97)
    ref = np.zeros((97, 12))
    np.add.at(ref, tok.ravel(), dx0)
    assert np.max(np.abs(dwte - ref)) < 1e-14
    assert np.max(np.abs(dwpe - dx0.reshape(3, 20, 12).sum(0))) < 1e-14
    # conservation: all of dx0 lands in dwte
    assert abs(dwte.sum() - dx0.sum()) < 1e-11


def test_linear_matches_matmul():
    rng = np.random.default_rng(7)
    X = rng.standard_normal((13, 7))
    W = rng.standard_normal((5, 7))
    b = rng.standard_normal(5)
    assert np.max(np.abs(oracle.linear_fwd(X, W, b) - (X @ W.T + b))) < 1e-13
    dY = rng.standard_normal((13, 5))
    dX, dW, db = oracle.linear_bwd(dY, X, W)
    assert np.max(np.abs(dX - dY @ W)) < 1e-13
    assert np.max(np.abs(dW - dY.T @ X)) < 1e-13
    assert np.max(np.abs(db - dY.sum(0))) < 1e-13


# --------------------------------------------------------------------------
# Gradients: central finite differences on every parameter of tiny shapes
# --------------------------------------------------------------------------
@pytest.mark.parametrize("cfg", [MICRO, MICRO_UNTIED], ids=["tied", "untied"])
def test_finite_differences_every_parameter(cfg):
    p = rand_params(cfg, 11, scale=10.0)
    tok, tgt = synth.micro_batch(2, cfg.T, cfg.V, dist="uniform", index=5)
    loss, g = oracle.forward_backward(cfg, p, tok, tgt)
    h = 1e-6
    fd = np.zeros_like(p)
    for i in range(p.size):
        pp = p.copy()
        pp[i] += h
        lp = oracle.forward(cfg, pp, tok, tgt, attn_mode=0)
        pp[i] -= 2 * h
        lm = oracle.forward(cfg, pp, tok, tgt, attn_mode=0)
        fd[i] = (lp - lm) / (2 * h)
    # central differences carry O(h^2) truncation and eps*loss/h ~ 3e-10 roundoff
    err = np.abs(fd - g)
    assert np.all(err <= 1e-6 * np.abs(g) + 1e-9), np.max(err)
    for t in oracle.tensors(cfg):
        sl = slice(t.offset, t.offset + t.size)
        assert np.linalg.norm(fd[sl] - g[sl]) <= 1e-6 * np.linalg.norm(g[sl]) + 1e-12, t.name


def test_full_model_matches_torch_autograd():
    """The whole forward/backward against a float64 model built from library
    routines (layer_norm, linear, SDPA, tanh-GELU, cross_entropy) and autograd."""
    for cfg in (oracle.Config(2, 2, 32, 16, 29, 1, 1), oracle.Config(2, 4, 32, 16, 29, 0, 0)):
        p = rand_params(cfg, 21)
        tok, tgt = synth.micro_batch(3, cfg.T, cfg.V, dist="uniform", index=2)
        loss, g = oracle.forward_backward(cfg, p, tok, tgt)
        tens = oracle.tensors(cfg)
        P = {t.name: torch.tensor(p[t.offset:t.offset + t.size].reshape(t.shape), requires_grad=True) for t in tens}
        B, T, C, NH = 3, cfg.T, cfg.C, cfg.H
        x = P["wte"][torch.from_numpy(tok).long()] + P["wpe"][:T]
        for l in range(cfg.L):
            pre = f"h{l}."
            hh = F.layer_norm(x, (C,), P[pre + "ln1_g"], P[pre + "ln1_b"], 1e-5)
            qkv = F.linear(hh, P[pre + "qkv_w"], P.get(pre + "qkv_b"))
            q, k, v = (qkv[..., i * C:(i + 1) * C].view(B, T, NH, C // NH).transpose(1, 2) for i in range(3))
            y = F.scaled_dot_product_attention(q, k, v, is_causal=True).transpose(1, 2).reshape(B, T, C)
            x = x + F.linear(y, P[pre + "ao_w"], P[pre + "ao_b"])
            hh = F.layer_norm(x, (C,), P[pre + "ln2_g"], P[pre + "ln2_b"], 1e-5)
            x = x + F.linear(F.gelu(F.linear(hh, P[pre + "fc_w"], P[pre + "fc_b"]), approximate="tanh"),
                             P[pre + "pj_w"], P[pre + "pj_b"])
        xf = F.layer_norm(x, (C,), P["lnf_g"], P["lnf_b"], 1e-5)
        logits = F.linear(xf, P["wte"] if cfg.tied else P["head_w"])
        ref = F.cross_entropy(logits.view(-1, cfg.V), torch.from_numpy(tgt).long().view(-1))
        ref.backward()
        assert abs(loss - ref.item()) < 1e-12
        for t in tens:
            gr = P[t.name].grad.numpy().ravel()
            mine = g[t.offset:t.offset + t.size]
            assert np.max(np.abs(mine - gr)) <= 1e-12 * max(1.0, np.max(np.abs(gr))), t.name


def test_accumulation_equals_big_batch():
    cfg = oracle.Config(2, 2, 32, 16, 29, 1, 1)
    p = rand_params(cfg, 8)
    toks, tgts, grads = [], [], []
    for m in range(4):
        tok, tgt = synth.micro_batch(2, cfg.T, cfg.V, index=m, dist="uniform")
        toks.append(tok)
        tgts.append(tgt)
        grads.append(oracle.forward_backward(cfg, p, tok, tgt)[1])
    G = sum(grads) / 4
    _, Gbig = oracle.forward_backward(cfg, p, np.concatenate(toks), np.concatenate(tgts))
    assert np.max(np.abs(G - Gbig)) <= 1e-10 * np.max(np.abs(Gbig))


def test_key_bias_gradient_vanishes():
    """Adding q.b_k to every score of a row leaves the softmax unchanged, so the
    gradient of the key third of the QKV bias is identically zero while the query
    and value parts are not."""
    p = rand_params(TINY, 15)
    tok, tgt = batch(TINY, 2)
    _, g = oracle.forward_backward(TINY, p, tok, tgt)
    C = TINY.C
    for t in oracle.tensors(TINY):
        if t.name.endswith("qkv_b"):
            gb = g[t.offset:t.offset + t.size]
            scale = np.max(np.abs(gb))
            assert np.max(np.abs(gb[C:2 * C])) <= 1e-12 * scale
            assert np.max(np.abs(gb[:C])) > 1e-6 * scale and np.max(np.abs(gb[2 * C:])) > 1e-3 * scale


def test_tying_gradient_is_sum_of_embedding_and_head_parts():
    tied = oracle.Config(2, 2, 16, 8, 23, 1, 1)
    untied = oracle.Config(2, 2, 16, 8, 23, 0, 1)
    pt = rand_params(tied, 9)
    tu = {t.name: t for t in oracle.tensors(untied)}
    tt = {t.name: t for t in oracle.tensors(tied)}
    pu = np.zeros(oracle.num_params(untied))
    for name, t in tt.items():
        pu[tu[name].offset:tu[name].offset + t.size] = pt[t.offset:t.offset + t.size]
    w = tt["wte"]
    pu[tu["head_w"].offset:tu["head_w"].offset + w.size] = pt[w.offset:w.offset + w.size]
    tok, tgt = synth.micro_batch(2, 8, 23, dist="uniform")
    lt, gt = oracle.forward_backward(tied, pt, tok, tgt)
    lu, gu = oracle.forward_backward(untied, pu, tok, tgt)
    assert abs(lt - lu) < 1e-14
    emb = gu[tu["wte"].offset:tu["wte"].offset + w.size]
    head = gu[tu["head_w"].offset:tu["head_w"].offset + w.size]
    assert np.max(np.abs(gt[w.offset:w.offset + w.size] - (emb + head))) < 1e-15
    assert np.max(np.abs(head)) > 0 and np.max(np.abs(emb)) > 0


# --------------------------------------------------------------------------
# Optimizer
# --------------------------------------------------------------------------
def test_adamw_first_step_closed_form(golden):
    cfg = oracle.Config(2, 2, 16, 8, 23, 1, 1)
    rng = np.random.default_rng(10)
    p0 = rand_params(cfg, 12)
    n = p0.size
    for gscale in (1e-3, 10.0):  # unclipped and clipped
        G = rng.standard_normal(n) * gscale / math.sqrt(n)
        lr, wd = golden["peak_lr"], golden["weight_decay"]
        p1, m1, v1, gn, clipped = oracle.adamw_step(cfg, p0, G, np.zeros(n), np.zeros(n), 1, lr, wd,
                                                    want_clipped=True)
        assert abs(gn - np.linalg.norm(G)) < 1e-12 * max(1, gn)
        if gn > 1:
            assert abs(np.linalg.norm(clipped) - 1.0) < 2e-6
        else:
            assert np.array_equal(clipped, G)
        decay = np.zeros(n)
        for t in oracle.tensors(cfg):
            decay[t.offset:t.offset + t.size] = 1.0 if len(t.shape) >= 2 else 0.0
        expect = p0 * (1 - lr * wd * decay) - lr * clipped / (np.abs(clipped) + 1e-8)
        assert np.max(np.abs(p1 - expect)) < 1e-15
        assert np.max(np.abs(m1 - 0.1 * clipped)) <= 1e-15 * np.max(np.abs(clipped))


def test_adamw_matches_torch_optimizer_three_steps(golden):
    cfg = oracle.Config(2, 2, 16, 8, 23, 1, 1)
    rng = np.random.default_rng(13)
    p = rand_params(cfg, 14)
    tens = oracle.tensors(cfg)
    tp = [torch.tensor(p[t.offset:t.offset + t.size].copy(), requires_grad=True) for t in tens]
    groups = [{"params": [x for x, t in zip(tp, tens) if len(t.shape) >= 2], "weight_decay": 0.1},
              {"params": [x for x, t in zip(tp, tens) if len(t.shape) < 2], "weight_decay": 0.0}]
    opt = torch.optim.AdamW(groups, lr=6e-4, betas=(0.9, 0.95), eps=1e-8)
    m = np.zeros_like(p)
    v = np.zeros_like(p)
    for step in range(1, 4):
        G = rng.standard_normal(p.size) * (0.3 if step != 2 else 0.001)
        for x, t in zip(tp, tens):
            x.grad = torch.tensor(G[t.offset:t.offset + t.size].copy())
        torch.nn.utils.clip_grad_norm_(tp, golden["grad_clip"])
        opt.step()
        p, m, v, _ = oracle.adamw_step(cfg, p, G, m, v, step, 6e-4, 0.1)
        ref = np.concatenate([x.detach().numpy() for x in tp])
        assert np.max(np.abs(p - ref)) < 1e-14


def test_decay_groups_are_the_2d_tensors():
    cfg = oracle.Config(12, 12, 768, 1024, 50257, 1, 1)
    tens = oracle.tensors(cfg)
    dec = [t for t in tens if t.decay]
    nodec = [t for t in tens if not t.decay]
    assert all(len(t.shape) == 2 for t in dec) and all(len(t.shape) == 1 for t in nodec)
    assert len(dec) == 2 + 4 * 12 and len(nodec) == 8 * 12 + 2
    C, F, V, T, L = 768, 3072, 50257, 1024, 12
    assert sum(t.size for t in dec) == V * C + T * C + L * (3 * C * C + C * C + 2 * F * C)
    assert sum(t.size for t in nodec) == L * (4 * C + 3 * C + C + F + C) + 2 * C


def test_canonical_order_and_offsets():
    cfg = oracle.Config(2, 2, 8, 5, 11, 0, 1)
    names = [t.name for t in oracle.tensors(cfg)]
    per = ["ln1_g", "ln1_b", "qkv_w", "qkv_b", "ao_w", "ao_b", "ln2_g", "ln2_b", "fc_w", "fc_b", "pj_w", "pj_b"]
    assert names == ["wte", "wpe"] + [f"h{l}.{n}" for l in range(2) for n in per] + ["lnf_g", "lnf_b", "head_w"]
    off = 0
    for t in oracle.tensors(cfg):
        assert t.offset == off
        off += t.size
    assert off == oracle.num_params(cfg)


def test_gpt2_124m_initial_loss_matches_a_library_model():
    """The oracle at the real 124M shape and initialisation (seed 42), against the same
    forward built from torch library routines in float64: the initial loss the GPU tests
    compare with is pinned at full width, depth and vocabulary (one 64-token Zipf
    sequence), not only on tiny shapes."""
    cfg = oracle.Config(12, 12, 768, 1024, 50257, 1, 1)
    p = oracle.init_params(cfg, 42).astype(np.float64)
    T = 64
    tok, tgt = synth.micro_batch(1, T, cfg.V, index=0)
    loss = oracle.forward(cfg, p, tok, tgt)
    P = {t.name: torch.from_numpy(p[t.offset:t.offset + t.size].reshape(t.shape)) for t in oracle.tensors(cfg)}
    C, NH = cfg.C, cfg.H
    with torch.no_grad():
        x = P["wte"][torch.from_numpy(tok).long()] + P["wpe"][:T]
        for l in range(cfg.L):
            pre = f"h{l}."
            hh = F.layer_norm(x, (C,), P[pre + "ln1_g"], P[pre + "ln1_b"], 1e-5)
            qkv = F.linear(hh, P[pre + "qkv_w"], P[pre + "qkv_b"])
            q, k, v = (qkv[..., i * C:(i + 1) * C].view(1, T, NH, C // NH).transpose(1, 2) for i in range(3))
            y = F.scaled_dot_product_attention(q, k, v, is_causal=True).transpose(1, 2).reshape(1, T, C)
            x = x + F.linear(y, P[pre + "ao_w"], P[pre + "ao_b"])
            hh = F.layer_norm(x, (C,), P[pre + "ln2_g"], P[pre + "ln2_b"], 1e-5)
            x = x + F.linear(F.gelu(F.linear(hh, P[pre + "fc_w"], P[pre + "fc_b"]), approximate="tanh"),
                             P[pre + "pj_w"], P[pre + "pj_b"])
        logits = F.linear(F.layer_norm(x, (C,), P["lnf_g"], P["lnf_b"], 1e-5), P["wte"])
        ref = F.cross_entropy(logits.view(-1, cfg.V), torch.from_numpy(tgt).long().view(-1)).item()
    assert abs(loss - ref) < 1e-9 * abs(ref), (loss, ref)
    # near ln V: the initial logits are nearly uniform apart from the tied head's small
    # preference for the input token itself
    assert abs(ref - np.log(cfg.V)) < 0.3, ref
