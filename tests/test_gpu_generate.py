"""Generation on the GPU: the sampler's indices equal the oracle's exactly on the same
fp32 logits, and the key/value-cache forward (prefill + decode steps) matches the float64
oracle's last-position logits within the bf16 bar (relative L2 <= 2e-2 per row, the
tolerance the training step's bf16 gradients are held to).
"""
import numpy as np
import pytest
import torch

import oracle
import train_step_b200 as tsb
from train_step_b200 import synth

pytestmark = pytest.mark.gpu

SMALL = tsb.Config(L=2, H=4, C=256, T=128, V=1000, tied=1, qkv_bias=1, dtype=tsb.BF16, B_max=4)


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def ocfg(c):
    return oracle.Config(c.L, c.H, c.C, c.T, c.V, c.tied, c.qkv_bias)


def _check_sampler(z, k, temp, top_p, u):
    zt = torch.from_numpy(np.ascontiguousarray(z, np.float32)).cuda()
    ut = torch.from_numpy(np.asarray(u, np.float64)).cuda()
    out = torch.empty(z.shape[0], dtype=torch.int32, device="cuda")
    tsb.sample_topk(zt, z.shape[1], k, temp, top_p, ut, out)
    got = out.cpu().numpy()
    want = [oracle.sample_topk(z[r], k, temp, top_p, float(u[r])) for r in range(z.shape[0])]
    assert got.tolist() == want, (k, temp, top_p)


@pytest.mark.parametrize("k,temp,top_p", [(1, 1.0, 1.0), (50, 1.0, 1.0), (50, 0.7, 0.9), (1024, 1.3, 1.0),
                                          (200, 1.0, 0.5), (1000, 2.0, 0.95)])
def test_sampler_exact_gpt2_vocab(k, temp, top_p):
    rng = np.random.default_rng(k)
    z = (rng.standard_normal((6, 50257)) * 3).astype(np.float32)
    _check_sampler(z, k, temp, top_p, rng.random(6))


def test_sampler_exact_heavy_ties():
    # few distinct values: the k-th largest value is shared by many indices across blocks
    rng = np.random.default_rng(3)
    for k in (1, 7, 100, 333, 1024):
        z = rng.integers(-3, 3, (4, 5000)).astype(np.float32)
        z[0, ::2] = 0.0
        z[0, 1::2] = -0.0
        _check_sampler(z, k, 1.0, 1.0, rng.random(4))


def test_sampler_ragged_and_small():
    rng = np.random.default_rng(9)
    for V in (1, 2, 17, 1023, 1025, 4097):
        z = (rng.standard_normal((3, V))).astype(np.float32)
        for k in sorted({1, min(V, 5), min(V, 1024)}):
            _check_sampler(z, k, 0.9, 1.0, rng.random(3))


def test_sampler_neg_inf_and_edges():
    rng = np.random.default_rng(11)
    z = (rng.standard_normal((4, 3000))).astype(np.float32)
    z[:, 100:2900] = -np.inf  # masked logits
    _check_sampler(z, 150, 1.0, 1.0, np.array([0.0, 0.25, 0.5, 0.999999]))
    with pytest.raises(tsb.Gpt2Error):
        _check_sampler(z, 0, 1.0, 1.0, rng.random(4))
    with pytest.raises(tsb.Gpt2Error):
        _check_sampler(z, 1025, 1.0, 1.0, rng.random(4))


def test_sampler_padded_rows():
    # rows with a stride above V (the library's padded vocabulary rows)
    rng = np.random.default_rng(4)
    full = (rng.standard_normal((5, 1064)) * 2).astype(np.float32)
    zt = torch.from_numpy(full).cuda()
    view = zt[:, :1000]
    u = rng.random(5)
    out = torch.empty(5, dtype=torch.int32, device="cuda")
    tsb.sample_topk(view, 1000, 40, 1.1, 1.0, torch.from_numpy(u).cuda(), out)
    assert out.cpu().tolist() == [oracle.sample_topk(full[r, :1000], 40, 1.1, 1.0, u[r]) for r in range(5)]


def _oracle_last_logits(cfg, p, seqs):
    seqs = np.ascontiguousarray(seqs, np.int32)
    B, T = seqs.shape
    _, logits = oracle.forward(ocfg(cfg), p, seqs, np.zeros_like(seqs), want_logits=True)
    return logits.reshape(B, T, cfg.V)[:, -1, :]


@pytest.mark.parametrize("cfg,B,T0,steps", [
    (SMALL, 3, 5, 4),
    (tsb.Config(L=2, H=2, C=128, T=96, V=777, tied=0, qkv_bias=0, dtype=tsb.BF16, B_max=3), 2, 1, 3),
])
def test_prefill_and_decode_match_oracle(cfg, B, T0, steps):
    m = tsb.GPT2(cfg, seed=13)
    p = m.get_params().astype(np.float64)
    rng = np.random.default_rng(2)
    seqs = rng.integers(0, cfg.V, (B, T0 + steps)).astype(np.int32)
    logits = m.prefill(torch.from_numpy(seqs[:, :T0]).cuda())
    assert m.kv_length == T0
    ref = _oracle_last_logits(cfg, p, seqs[:, :T0])
    for b in range(B):
        assert rel_l2(logits[b].cpu().numpy(), ref[b]) <= 2e-2
    for s in range(steps):
        logits = m.decode_step(torch.from_numpy(seqs[:, T0 + s].copy()))
        assert m.kv_length == T0 + s + 1
        ref = _oracle_last_logits(cfg, p, seqs[:, :T0 + s + 1])
        for b in range(B):
            e = rel_l2(logits[b].cpu().numpy(), ref[b])
            assert e <= 2e-2, (s, b, e)
    m.close()


def test_decode_agrees_with_prefill_of_whole_sequence():
    # the cached path and a fresh forward of the full sequence give the same last logits
    m = tsb.GPT2(SMALL, seed=21)
    seqs = torch.from_numpy(np.random.default_rng(8).integers(0, SMALL.V, (4, 40)).astype(np.int32)).cuda()
    m.prefill(seqs[:, :30].contiguous())
    for s in range(30, 40):
        dec = m.decode_step(seqs[:, s].contiguous()).cpu().numpy()
    full = tsb.GPT2(SMALL, seed=21)
    pre = full.prefill(seqs).cpu().numpy()
    for b in range(4):
        assert rel_l2(dec[b], pre[b]) <= 1e-2
    m.close()
    full.close()


def test_generate_draws_match_oracle_sampler_and_cache_limit():
    m = tsb.GPT2(SMALL, seed=17)
    prompt = torch.from_numpy(np.random.default_rng(1).integers(0, SMALL.V, (2, 6)).astype(np.int32)).cuda()
    k, temp, top_p = 40, 0.9, 0.95
    u = np.random.default_rng(123).random((5, 2))
    logits = m.prefill(prompt)
    idx = torch.empty(2, dtype=torch.int32, device="cuda")
    drawn = []
    for s in range(5):
        z = logits.cpu().numpy()
        m.sample_topk(logits, k, temp, top_p, torch.from_numpy(u[s].copy()).cuda(), out=idx)
        assert idx.cpu().tolist() == [oracle.sample_topk(z[r], k, temp, top_p, u[s, r]) for r in range(2)]
        drawn.append(idx.cpu().numpy().copy())
        logits = m.decode_step(idx)
    # generate() with the same seed draws the same u and so the same tokens
    g = tsb.GPT2(SMALL, seed=17).generate(prompt, 5, k=k, temperature=temp, top_p=top_p, seed=123)
    assert np.array_equal(g[:, 6:].cpu().numpy(), np.stack(drawn, 1))
    # the cache holds T positions: decoding past them is an error, not a fault
    while m.kv_length < SMALL.T:
        m.decode_step(idx)
    with pytest.raises(tsb.Gpt2Error):
        m.decode_step(idx)
    m.close()


def test_generation_rejects_fp32_models():
    m = tsb.GPT2(tsb.Config(L=1, H=2, C=128, T=16, V=50, dtype=tsb.FP32, B_max=2), seed=1)
    with pytest.raises(tsb.Gpt2Error):
        m.prefill(torch.zeros(1, 4, dtype=torch.int32, device="cuda"))
    m.close()


def test_captured_step_equals_launch_by_launch():
    # the decode step replayed from its CUDA graph and the same kernels launched one by one
    # (profiling mode) give bit-identical logits and caches
    seqs = torch.from_numpy(np.random.default_rng(6).integers(0, SMALL.V, (3, 20)).astype(np.int32)).cuda()
    outs = []
    for profile in (False, True):
        m = tsb.GPT2(SMALL, seed=4)
        m.profile(profile)
        m.prefill(seqs[:, :12].contiguous())
        for s in range(12, 20):
            z = m.decode_step(seqs[:, s].contiguous())
        outs.append(z.cpu().numpy().copy())
        m.profile(False)
        m.close()
    assert np.array_equal(outs[0], outs[1])


def test_split_key_attention_many_splits():
    # B = 1 spreads each head's keys over up to 16 blocks; compare with the oracle at a
    # long context so that every split holds keys
    cfg = tsb.Config(L=1, H=2, C=128, T=512, V=300, tied=1, qkv_bias=1, dtype=tsb.BF16, B_max=1)
    m = tsb.GPT2(cfg, seed=8)
    p = m.get_params().astype(np.float64)
    seq = np.random.default_rng(12).integers(0, cfg.V, (1, 400)).astype(np.int32)
    m.prefill(torch.from_numpy(seq[:, :397].copy()).cuda())
    for s in range(397, 400):
        z = m.decode_step(torch.from_numpy(seq[:, s].copy())).cpu().numpy()
    ref = _oracle_last_logits(cfg, p, seq)
    assert rel_l2(z[0], ref[0]) <= 2e-2
    m.close()


def _dev(a, dtype):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(dtype).cuda()


def _g64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("B,N,K", [(1, 2304, 768), (5, 770, 256), (16, 3072, 768), (16, 768, 3072), (3, 1001, 128),
                                   (16, 50257, 768)])
def test_gemv_epilogues_match_oracle(B, N, K):
    rng = np.random.default_rng(N + K + B)
    x = _dev(rng.standard_normal((B, K)), torch.bfloat16)
    W = _dev(rng.standard_normal((N, K)) * 0.05, torch.bfloat16)
    bias = _dev(rng.standard_normal(N), torch.float32)
    resid = _dev(rng.standard_normal((B, N)), torch.float32)
    D = oracle.linear_fwd(_g64(x), _g64(W))
    kw = dict(B=B, N=N, K=K)
    o0 = torch.empty(B, N, dtype=torch.bfloat16, device="cuda")
    tsb.gemv(x, W, o0, epilogue=tsb.EPI_BIAS, bias=bias, **kw)
    assert rel_l2(_g64(o0), D + _g64(bias)) < 4e-3
    o1 = torch.empty_like(o0)
    tsb.gemv(x, W, o1, epilogue=tsb.EPI_BIAS_GELU, bias=bias, **kw)
    assert rel_l2(_g64(o1), oracle.gelu_fwd(D + _g64(bias))) < 5e-3
    o2 = torch.empty(B, N, dtype=torch.float32, device="cuda")
    tsb.gemv(x, W, o2, epilogue=tsb.EPI_RESID, bias=bias, resid=resid, ldr=N, **kw)
    assert rel_l2(_g64(o2), D + _g64(bias) + _g64(resid)) < 1e-5
    o4 = torch.empty(B, N, dtype=torch.float32, device="cuda")
    tsb.gemv(x, W, o4, epilogue=tsb.EPI_F32, **kw)
    assert rel_l2(_g64(o4), D) < 1e-5
    # LayerNorm applied on the fly to fp32 rows (the kernel rounds the normalised rows to bf16)
    xf = _dev(rng.standard_normal((B, K)) * 3 + 1, torch.float32)
    g = _dev(1 + 0.1 * rng.standard_normal(K), torch.float32)
    b = _dev(0.1 * rng.standard_normal(K), torch.float32)
    y, _, _ = oracle.layernorm_fwd(_g64(xf), _g64(g), _g64(b))
    tsb.gemv(xf, W, o4, epilogue=tsb.EPI_F32, ln_g=g, ln_b=b, **kw)
    assert rel_l2(_g64(o4), oracle.linear_fwd(y, _g64(W))) < 4e-3


def test_generation_token_range_errors():
    m = tsb.GPT2(SMALL, seed=2)
    bad = torch.full((2, 4), SMALL.V, dtype=torch.int32)
    with pytest.raises(tsb.Gpt2Error):
        m.prefill(bad)
    good = torch.randint(0, SMALL.V, (2, 4), dtype=torch.int32)
    m.prefill(good)
    with pytest.raises(tsb.Gpt2Error):
        m.decode_step(torch.tensor([0, -1], dtype=torch.int32))  # reported by the synchronisation
    m.decode_step(torch.tensor([1, 2], dtype=torch.int32))       # the handle stays usable
    with pytest.raises(tsb.Gpt2Error):
        m.decode_step(torch.tensor([1, 2, 3], dtype=torch.int32))  # B differs from the prefill's
    m.close()
