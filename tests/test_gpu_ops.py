"""Per-kernel parity of the CUDA library against the float64 oracle (GPU).

Each kernel is called through its C-ABI op entry point on seeded inputs and
compared element by element with the oracle's single-operation function on the
same (bf16-rounded where the kernel reads bf16) inputs. Shapes span several tiles
and a ragged tail.
"""
import math

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
    if nb == 0:
        return float(np.linalg.norm(a))
    return float(np.linalg.norm(a - b) / nb)


def g64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def randn(shape, seed, dtype=torch.bfloat16, scale=1.0):
    gen = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=gen, dtype=torch.float32) * scale).to(dtype).to(DEV)


# ---------------------------------------------------------------------------
# GEMM (tcgen05 bf16 path and fp32 SIMT path)
# ---------------------------------------------------------------------------
def operand(rows, cols, mn, seed, dtype):
    """Logical matrix [rows, cols] (contraction along cols) stored K-major
    ([rows][cols]) or MN-major ([cols][rows])."""
    logical = randn((rows, cols), seed, dtype)
    stored = logical.t().contiguous() if mn else logical.contiguous()
    ld = rows if mn else cols
    return logical, stored, ld


GEMM_SHAPES = [(300, 384, 200), (256, 128, 64), (128, 520, 136), (1000, 768, 768), (296, 2304, 1024), (15, 256, 136)]
MAJORS = [(False, False), (False, True), (True, True)]


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
@pytest.mark.parametrize("a_mn,b_mn", MAJORS)
def test_gemm_bf16_store_and_accumulate(M, N, K, a_mn, b_mn):
    if a_mn and M % 8:
        M += 8 - M % 8
    A, As, lda = operand(M, K, a_mn, 1, torch.bfloat16)
    B, Bs, ldb = operand(N, K, b_mn, 2, torch.bfloat16)
    ref = oracle.linear_fwd(g64(A), g64(B))
    out = torch.zeros(M, N, dtype=torch.float32, device=DEV)
    tsb.gemm(As, Bs, out, M=M, N=N, K=K, lda=lda, ldb=ldb, ldo=N, a_mn=a_mn, b_mn=b_mn, epilogue=tsb.EPI_F32)
    torch.cuda.synchronize()
    assert rel_l2(g64(out), ref) < 1e-5
    # accumulate on top of an existing value, and split-K
    base = randn((M, N), 3, torch.float32)
    out2 = base.clone()
    tsb.gemm(As, Bs, out2, M=M, N=N, K=K, lda=lda, ldb=ldb, ldo=N, a_mn=a_mn, b_mn=b_mn, epilogue=tsb.EPI_F32,
             accumulate=True, ksplit=3 if K >= 192 else 1)
    torch.cuda.synchronize()
    assert rel_l2(g64(out2), ref + g64(base)) < 1e-5


@pytest.mark.parametrize("M,N,K", [(300, 384, 200), (1000, 3072, 768), (130, 136, 72)])
def test_gemm_bf16_epilogues(M, N, K):
    A = randn((M, K), 4, torch.bfloat16)
    W = randn((N, K), 5, torch.bfloat16, scale=0.5)
    bias = randn((N,), 6, torch.float32)
    D = oracle.linear_fwd(g64(A), g64(W))
    # 0: out = D + bias (bf16)
    out = torch.zeros(M, N, dtype=torch.bfloat16, device=DEV)
    tsb.gemm(A, W, out, M=M, N=N, K=K, lda=K, ldb=K, ldo=N, epilogue=tsb.EPI_BIAS, bias=bias)
    torch.cuda.synchronize()
    ref = D + g64(bias)
    assert rel_l2(g64(out), ref) < 4e-3
    # 1: u = D + bias, a = gelu(u)
    u = torch.zeros(M, N, dtype=torch.bfloat16, device=DEV)
    a = torch.zeros_like(u)
    tsb.gemm(A, W, u, M=M, N=N, K=K, lda=K, ldb=K, ldo=N, epilogue=tsb.EPI_BIAS_GELU, out2=a, ldo2=N, bias=bias)
    torch.cuda.synchronize()
    assert rel_l2(g64(u), ref) < 4e-3
    assert rel_l2(g64(a), oracle.gelu_fwd(ref)) < 5e-3
    # 2: out = resid + D + bias (fp32)
    res = randn((M, N), 7, torch.float32)
    o2 = torch.zeros(M, N, dtype=torch.float32, device=DEV)
    tsb.gemm(A, W, o2, M=M, N=N, K=K, lda=K, ldb=K, ldo=N, epilogue=tsb.EPI_RESID, bias=bias, aux=res, ld_aux=N)
    torch.cuda.synchronize()
    assert rel_l2(g64(o2), ref + g64(res)) < 1e-5
    # 3: out = D * gelu'(aux)
    ua = randn((M, N), 8, torch.bfloat16)
    o3 = torch.zeros(M, N, dtype=torch.bfloat16, device=DEV)
    tsb.gemm(A, W, o3, M=M, N=N, K=K, lda=K, ldb=K, ldo=N, epilogue=tsb.EPI_DGELU, aux=ua, ld_aux=N)
    torch.cuda.synchronize()
    assert rel_l2(g64(o3), oracle.gelu_bwd(g64(ua), D)) < 5e-3


@pytest.mark.parametrize("M,N,K", [(300, 520, 200), (130, 256, 72), (1000, 768, 768), (512, 2304, 1024)])
@pytest.mark.parametrize("a_mn,b_mn", MAJORS)
def test_gemm_bf16_pair_tiles(M, N, K, a_mn, b_mn):
    """256 x 256 tiles computed by a 2-CTA cluster (M = 256 MMAs across both SMs), forced
    through the timing entry point: every epilogue, ragged M / N tails (the second CTA's
    rows partly or wholly past M), and a split-K fp32 store."""
    if a_mn and M % 8:
        M += 8 - M % 8
    A, As, lda = operand(M, K, a_mn, 11, torch.bfloat16)
    B, Bs, ldb = operand(N, K, b_mn, 12, torch.bfloat16)
    D = oracle.linear_fwd(g64(A), g64(B))
    bias = randn((N,), 13, torch.float32)
    kw = dict(M=M, N=N, K=K, lda=lda, ldb=ldb, ldo=N, a_mn=a_mn, b_mn=b_mn, bn=256, pair=1, iters=1)
    out = torch.zeros(M, N, dtype=torch.float32, device=DEV)
    tsb.gemm_bench(As, Bs, out, epilogue=tsb.EPI_F32, **kw)
    torch.cuda.synchronize()
    assert rel_l2(g64(out), D) < 1e-5
    if K >= 192:
        out.zero_()
        tsb.gemm_bench(As, Bs, out, epilogue=tsb.EPI_F32, ksplit=3, **kw)
        torch.cuda.synchronize()
        assert rel_l2(g64(out), D) < 1e-5
    ref = D + g64(bias)
    o0 = torch.zeros(M, N, dtype=torch.bfloat16, device=DEV)
    tsb.gemm_bench(As, Bs, o0, epilogue=tsb.EPI_BIAS, bias=bias, **kw)
    u = torch.zeros(M, N, dtype=torch.bfloat16, device=DEV)
    a = torch.zeros_like(u)
    tsb.gemm_bench(As, Bs, u, epilogue=tsb.EPI_BIAS_GELU, out2=a, ldo2=N, bias=bias, **kw)
    res = randn((M, N), 14, torch.float32)
    o2 = torch.zeros(M, N, dtype=torch.float32, device=DEV)
    tsb.gemm_bench(As, Bs, o2, epilogue=tsb.EPI_RESID, bias=bias, aux=res, ld_aux=N, **kw)
    ua = randn((M, N), 15, torch.bfloat16)
    o3 = torch.zeros(M, N, dtype=torch.bfloat16, device=DEV)
    tsb.gemm_bench(As, Bs, o3, epilogue=tsb.EPI_DGELU, aux=ua, ld_aux=N, **kw)
    torch.cuda.synchronize()
    assert rel_l2(g64(o0), ref) < 4e-3
    assert rel_l2(g64(u), ref) < 4e-3
    assert rel_l2(g64(a), oracle.gelu_fwd(ref)) < 5e-3
    assert rel_l2(g64(o2), ref + g64(res)) < 1e-5
    assert rel_l2(g64(o3), oracle.gelu_bwd(g64(ua), D)) < 5e-3


@pytest.mark.parametrize("a_mn,b_mn", MAJORS)
@pytest.mark.parametrize("epi", [0, 1, 2, 3, 4])
def test_gemm_fp32_simt(a_mn, b_mn, epi):
    M, N, K = 130, 70, 45
    A, As, lda = operand(M, K, a_mn, 9, torch.float32)
    B, Bs, ldb = operand(N, K, b_mn, 10, torch.float32)
    bias = randn((N,), 11, torch.float32)
    aux = randn((M, N), 12, torch.float32)
    D = oracle.linear_fwd(g64(A), g64(B))
    out = torch.zeros(M, N, dtype=torch.float32, device=DEV)
    out2 = torch.zeros_like(out)
    tsb.gemm(As, Bs, out, M=M, N=N, K=K, lda=lda, ldb=ldb, ldo=N, a_mn=a_mn, b_mn=b_mn, epilogue=epi, out2=out2,
             ldo2=N, bias=bias if epi in (0, 1, 2) else None, aux=aux if epi in (2, 3) else None, ld_aux=N)
    torch.cuda.synchronize()
    if epi in (0, 1):
        assert rel_l2(g64(out), D + g64(bias)) < 1e-6
        if epi == 1:
            assert rel_l2(g64(out2), oracle.gelu_fwd(D + g64(bias))) < 1e-6
    elif epi == 2:
        assert rel_l2(g64(out), D + g64(bias) + g64(aux)) < 1e-6
    elif epi == 3:
        assert rel_l2(g64(out), oracle.gelu_bwd(g64(aux), D)) < 1e-6
    else:
        assert rel_l2(g64(out), D) < 1e-6


# ---------------------------------------------------------------------------
# LayerNorm
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("N,C", [(1000, 768), (77, 1600), (512, 128), (16384, 768), (3001, 1024), (5, 768),
                                 (2371, 256), (9999, 1024), (9473, 256)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_layernorm_fwd_bwd(N, C, dtype):
    x = randn((N, C), 20, torch.float32, scale=2.0) + 0.5
    g = randn((C,), 21, torch.float32) * 0.3 + 1.0
    b = randn((C,), 22, torch.float32) * 0.1
    y = torch.zeros(N, C, dtype=dtype, device=DEV)
    mean = torch.zeros(N, device=DEV)
    rstd = torch.zeros(N, device=DEV)
    tsb.layernorm_fwd(x, g, b, y, mean, rstd)
    torch.cuda.synchronize()
    ry, rm, rr = oracle.layernorm_fwd(g64(x), g64(g), g64(b))
    tol = 4e-3 if dtype == torch.bfloat16 else 1e-6
    assert rel_l2(g64(y), ry) < tol
    assert rel_l2(g64(mean), rm) < 1e-6 and rel_l2(g64(rstd), rr) < 1e-6
    dy = randn((N, C), 23, torch.float32)
    dres0 = randn((N, C), 24, torch.float32)
    dres = dres0.clone()
    dres_act = torch.zeros(N, C, dtype=dtype, device=DEV) if dtype == torch.bfloat16 else None
    dg = torch.ones(C, device=DEV)
    db = torch.ones(C, device=DEV)
    tsb.layernorm_bwd(dy, x, g, mean, rstd, dres, dres_act, dg, db, accumulate=True, accumulate_params=True,
                      dtype=tsb.BF16 if dtype == torch.bfloat16 else tsb.FP32)
    torch.cuda.synchronize()
    rdx, rdg, rdb = oracle.layernorm_bwd(g64(dy), g64(x), g64(g), g64(mean), g64(rstd))
    assert rel_l2(g64(dres), rdx + g64(dres0)) < 1e-5
    if dres_act is not None:
        assert rel_l2(g64(dres_act), rdx + g64(dres0)) < 4e-3
    assert rel_l2(g64(dg), rdg + 1) < 1e-5 and rel_l2(g64(db), rdb + 1) < 1e-5


@pytest.mark.parametrize("N,C", [(1000, 768), (3001, 1024), (77, 1600)])
def test_layernorm_bwd_overwrite(N, C):
    """accumulate = 0: dres is overwritten (never read), the parameter grads too."""
    x = randn((N, C), 25, torch.float32, scale=2.0) - 0.25
    g = randn((C,), 26, torch.float32) * 0.3 + 1.0
    b = torch.zeros(C, device=DEV)
    y = torch.zeros(N, C, dtype=torch.bfloat16, device=DEV)
    mean = torch.zeros(N, device=DEV)
    rstd = torch.zeros(N, device=DEV)
    tsb.layernorm_fwd(x, g, b, y, mean, rstd)
    dy = randn((N, C), 27, torch.float32)
    dres = torch.full((N, C), float("nan"), device=DEV)
    dres_act = torch.zeros(N, C, dtype=torch.bfloat16, device=DEV)
    dg = torch.full((C,), float("nan"), device=DEV)
    db = torch.full((C,), float("nan"), device=DEV)
    tsb.layernorm_bwd(dy, x, g, mean, rstd, dres, dres_act, dg, db, accumulate=False, accumulate_params=False,
                      dtype=tsb.BF16)
    torch.cuda.synchronize()
    rdx, rdg, rdb = oracle.layernorm_bwd(g64(dy), g64(x), g64(g), g64(mean), g64(rstd))
    assert rel_l2(g64(dres), rdx) < 1e-5
    assert rel_l2(g64(dres_act), rdx) < 4e-3
    assert rel_l2(g64(dg), rdg) < 1e-5 and rel_l2(g64(db), rdb) < 1e-5


# ---------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------
def _attention_bwd_stored(qkv, out, dout, lse, dqkv, B, T, NH, hd):
    """The training step's backward: dS^T tiles kept in a workspace, dQ computed from them.
    The workspace starts as NaN so that a tile the dQ pass reads but nobody wrote shows."""
    nbytes = tsb.attention_ds_bytes(B, T, NH)
    nqb = (T + 127) // 128
    assert nbytes == B * NH * nqb * nqb * 128 * 128 * 2
    ds = torch.full((nbytes // 2,), float("nan"), dtype=torch.bfloat16, device=DEV)
    tsb.attention_bwd_stored(qkv, out, dout, lse, dqkv, ds, B, T, NH, hd)
    return ds


@pytest.mark.parametrize("stored", [False, True])
@pytest.mark.parametrize("B,T,NH", [(2, 200, 2), (1, 256, 3), (2, 64, 1), (1, 1024, 2), (1, 17, 2), (3, 300, 1),
                                    (1, 129, 2), (1, 385, 1), (2, 512, 2), (1, 1024, 16), (1, 640, 25)])
def test_attention_bf16(B, T, NH, stored):
    hd = 64
    C = NH * hd
    qkv = randn((B * T, 3 * C), 30, torch.bfloat16)
    out = torch.zeros(B * T, C, dtype=torch.bfloat16, device=DEV)
    lse = torch.zeros(B, NH, T, device=DEV)
    tsb.attention_fwd(qkv, out, lse, B, T, NH, hd)
    torch.cuda.synchronize()
    ro, rl = oracle.attention_fwd(g64(qkv), B, T, NH, hd, mode=0)
    assert rel_l2(g64(out), ro) < 1e-2
    assert np.max(np.abs(g64(lse) - rl)) < 2e-3
    dout = randn((B * T, C), 31, torch.bfloat16)
    dqkv = torch.zeros_like(qkv)
    tsb.attention_bwd(qkv, out, dout, lse, dqkv, B, T, NH, hd)
    if stored:
        recomputed = dqkv.clone()
        dqkv.fill_(float("nan"))
        _attention_bwd_stored(qkv, out, dout, lse, dqkv, B, T, NH, hd)
    torch.cuda.synchronize()
    rd = oracle.attention_bwd(g64(qkv), g64(dout), B, T, NH, hd)
    got = g64(dqkv)
    for part in range(3):
        sl = slice(part * C, (part + 1) * C)
        assert rel_l2(got[:, sl], rd[:, sl]) < 2e-2, part
    if stored:
        # dK and dV come from the same kernel arithmetic in both forms
        assert torch.equal(dqkv[:, C:], recomputed[:, C:])


def test_attention_bwd_stored_rejects_a_bad_workspace():
    """The stored-dS entry point: no workspace, or one that is not 16-byte aligned, is a
    configuration error reported before any dS tile is written; the next call works."""
    B, T, NH, hd = 1, 256, 2, 64
    C = NH * hd
    qkv = randn((B * T, 3 * C), 35, torch.bfloat16)
    out = torch.zeros(B * T, C, dtype=torch.bfloat16, device=DEV)
    lse = torch.zeros(B, NH, T, device=DEV)
    tsb.attention_fwd(qkv, out, lse, B, T, NH, hd)
    dout = randn((B * T, C), 36, torch.bfloat16)
    dqkv = torch.zeros_like(qkv)
    with pytest.raises(tsb.Gpt2Error) as e:
        tsb.attention_bwd_stored(qkv, out, dout, lse, dqkv, None, B, T, NH, hd)
    assert e.value.code == -1
    nbytes = tsb.attention_ds_bytes(B, T, NH)
    raw = torch.zeros(nbytes // 2 + 8, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(tsb.Gpt2Error) as e:
        tsb.attention_bwd_stored(qkv, out, dout, lse, dqkv, raw[1:], B, T, NH, hd)  # 2-byte offset
    assert e.value.code == -1
    ref = torch.zeros_like(qkv)
    tsb.attention_bwd(qkv, out, dout, lse, ref, B, T, NH, hd)
    _attention_bwd_stored(qkv, out, dout, lse, dqkv, B, T, NH, hd)
    torch.cuda.synchronize()
    assert torch.equal(dqkv[:, C:], ref[:, C:])
    assert rel_l2(g64(dqkv[:, :C]), g64(ref[:, :C])) < 1e-2


def test_attention_bf16_running_max_rebase():
    """Scores that grow by ~12 (log2 units) per 64 keys on odd query rows and stay flat
    on even rows: the odd rows re-base their running maximum (rescaling their output
    accumulator row) on every unit while their even neighbours in the same warp do not.
    Forward only: on rows this peaked, dS = P (dP - D) cancels to below the bf16 rounding
    of the stored output that D is computed from, so the backward has no meaningful
    tolerance here (and it has no running maximum)."""
    B, T, NH, hd = 1, 512, 2, 64
    C = NH * hd
    gen = torch.Generator().manual_seed(40)
    qkv = torch.zeros(B * T, 3 * C)
    t = torch.arange(T, dtype=torch.float32)
    for h in range(NH):
        qkv[:, h * hd] = torch.where(t % 2 == 1, 32.0, 0.0)    # q_t = a_t e0
        qkv[:, C + h * hd] = 33.0 * t / T                       # k_j = 33 j / T e0
        qkv[:, 2 * C + h * hd:2 * C + (h + 1) * hd] = torch.randn(T, hd, generator=gen)
    qkv = qkv.to(torch.bfloat16).to(DEV)
    out = torch.zeros(B * T, C, dtype=torch.bfloat16, device=DEV)
    lse = torch.zeros(B, NH, T, device=DEV)
    tsb.attention_fwd(qkv, out, lse, B, T, NH, hd)
    torch.cuda.synchronize()
    ro, rl = oracle.attention_fwd(g64(qkv), B, T, NH, hd, mode=0)
    assert rel_l2(g64(out), ro) < 1e-2
    assert np.max(np.abs(g64(lse) - rl) / np.maximum(1.0, np.abs(rl))) < 1e-3


def test_attention_bf16_full_size_sampled_heads():
    """The training step's launch (B = 16, T = 1024, 12 heads of 64, as the benchmark runs
    it), checked against the oracle on sampled (sequence, head) pairs: the oracle runs on
    each pair's own columns, which is exact since heads and sequences are independent."""
    B, T, NH, hd = 16, 1024, 12, 64
    C = NH * hd
    qkv = randn((B * T, 3 * C), 33, torch.bfloat16)
    out = torch.zeros(B * T, C, dtype=torch.bfloat16, device=DEV)
    lse = torch.zeros(B, NH, T, device=DEV)
    tsb.attention_fwd(qkv, out, lse, B, T, NH, hd)
    dout = randn((B * T, C), 34, torch.bfloat16)
    dqkv = torch.zeros_like(qkv)
    tsb.attention_bwd(qkv, out, dout, lse, dqkv, B, T, NH, hd)
    dqkv_s = torch.zeros_like(qkv)
    _attention_bwd_stored(qkv, out, dout, lse, dqkv_s, B, T, NH, hd)
    torch.cuda.synchronize()
    assert torch.equal(dqkv_s[:, C:], dqkv[:, C:])
    assert rel_l2(g64(dqkv_s[:, :C]), g64(dqkv[:, :C])) < 1e-2
    q3 = g64(qkv).reshape(B, T, 3, NH, hd)
    o3 = g64(out).reshape(B, T, NH, hd)
    d3 = g64(dout).reshape(B, T, NH, hd)
    g3 = g64(dqkv).reshape(B, T, 3, NH, hd)
    for b, h in [(0, 0), (7, 5), (15, 11), (3, 9)]:
        qkv1 = q3[b, :, :, h, :].reshape(T, 3 * hd)
        ro, rl = oracle.attention_fwd(qkv1, 1, T, 1, hd, mode=0)
        assert rel_l2(o3[b, :, h, :], ro) < 1e-2, (b, h)
        assert np.max(np.abs(g64(lse[b, h]) - rl[0, 0])) < 2e-3, (b, h)
        rd = oracle.attention_bwd(qkv1, d3[b, :, h, :], 1, T, 1, hd).reshape(T, 3, hd)
        for part in range(3):
            assert rel_l2(g3[b, :, part, h, :], rd[:, part]) < 2e-2, (b, h, part)
        # the stored-dS form's dQ (the training step's) against the oracle too
        gs = g64(dqkv_s[:, :C]).reshape(B, T, NH, hd)
        assert rel_l2(gs[b, :, h, :], rd[:, 0]) < 2e-2, (b, h)


@pytest.mark.parametrize("B,T,NH,hd", [(2, 70, 2, 32), (1, 64, 4, 64), (2, 33, 1, 128)])
def test_attention_fp32(B, T, NH, hd):
    C = NH * hd
    qkv = randn((B * T, 3 * C), 32, torch.float32)
    out = torch.zeros(B * T, C, device=DEV)
    lse = torch.zeros(B, NH, T, device=DEV)
    tsb.attention_fwd(qkv, out, lse, B, T, NH, hd)
    dout = randn((B * T, C), 33, torch.float32)
    dqkv = torch.zeros_like(qkv)
    tsb.attention_bwd(qkv, out, dout, lse, dqkv, B, T, NH, hd)
    torch.cuda.synchronize()
    ro, rl = oracle.attention_fwd(g64(qkv), B, T, NH, hd, mode=0)
    assert rel_l2(g64(out), ro) < 1e-5
    assert np.max(np.abs(g64(lse) - rl)) < 1e-5
    rd = oracle.attention_bwd(g64(qkv), g64(dout), B, T, NH, hd)
    assert rel_l2(g64(dqkv), rd) < 1e-5


# ---------------------------------------------------------------------------
# embedding
# ---------------------------------------------------------------------------
def test_embedding_fwd_bit_exact():
    B, T, C, V = 3, 100, 768, 50257
    tok, _ = synth.micro_batch(B, T, V)
    wte = randn((V, C), 40, torch.float32, 0.02)
    wpe = randn((T, C), 41, torch.float32, 0.02)
    x0 = torch.zeros(B * T, C, device=DEV)
    tsb.embedding_fwd(torch.from_numpy(tok).to(DEV), wte, wpe, x0)
    ref = oracle.embedding_fwd(tok, g64(wte), g64(wpe)).astype(np.float32)
    assert np.array_equal(x0.cpu().numpy(), ref)


@pytest.mark.parametrize("N", [1, 777, 16384, 32768])
def test_token_buckets_exact(N):
    V = 50257
    tok = synth.zipf_ids(99 + N, N, V)
    td = torch.from_numpy(tok).to(DEV)
    sp = torch.zeros(N, dtype=torch.int32, device=DEV)
    sid = torch.zeros(N, dtype=torch.int32, device=DEV)
    sst = torch.zeros(N + 1, dtype=torch.int32, device=DEV)
    nseg = tsb.token_buckets(td, V, sp, sid, sst)
    counts, offsets, pos = oracle.token_buckets(tok, V)
    ids = np.nonzero(counts)[0]
    assert nseg == len(ids)
    assert np.array_equal(sp.cpu().numpy(), pos)
    assert np.array_equal(sid.cpu().numpy()[:nseg], ids)
    assert np.array_equal(sst.cpu().numpy()[:nseg + 1], np.append(offsets[ids], N))


@pytest.mark.parametrize("B,T,C", [(4, 1024, 768), (16, 1024, 768), (3, 50, 128)])
def test_embedding_bwd(B, T, C):
    V = 50257
    tok, _ = synth.micro_batch(B, T, V, index=3)
    dx0 = randn((B * T, C), 42, torch.float32)
    dwte0 = randn((V, C), 43, torch.float32, 0.01)
    dwpe0 = randn((T, C), 44, torch.float32, 0.01)
    dwte, dwpe = dwte0.clone(), dwpe0.clone()
    td = torch.from_numpy(tok).to(DEV)
    tsb.embedding_bwd(td, dx0, dwte, dwpe)
    torch.cuda.synchronize()
    rw, rp = oracle.embedding_bwd(tok, g64(dx0), V)
    assert rel_l2(g64(dwte) - g64(dwte0), rw) < 1e-6
    assert rel_l2(g64(dwpe) - g64(dwpe0), rp) < 1e-6
    # deterministic: a second run from the same start is bitwise identical
    dwte2, dwpe2 = dwte0.clone(), dwpe0.clone()
    tsb.embedding_bwd(td, dx0, dwte2, dwpe2)
    torch.cuda.synchronize()
    assert torch.equal(dwte, dwte2) and torch.equal(dwpe, dwpe2)


# ---------------------------------------------------------------------------
# cross-entropy
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("N,V,ld,dtype", [(300, 50257, 50304, torch.bfloat16), (64, 65, 128, torch.float32),
                                          (7, 65, 128, torch.bfloat16)])
def test_cross_entropy(N, V, ld, dtype):
    z = randn((N, ld), 50, dtype, scale=2.0)
    tgt = synth.zipf_ids(51, N, V) if V > 100 else synth.uniform_ids(51, N, V)
    zin = g64(z)
    rl = torch.zeros(N, device=DEV)
    tsb.cross_entropy(z, V, torch.from_numpy(tgt).to(DEV), 1.0 / N, rl)
    torch.cuda.synchronize()
    tot, rrow, rdl = oracle.cross_entropy(zin, V, tgt, scale=1.0 / N)
    tol = 2e-4 if dtype == torch.bfloat16 else 1e-6
    assert np.max(np.abs(g64(rl) - rrow)) < tol * max(1.0, np.max(np.abs(rrow)))
    assert rel_l2(g64(z), rdl) < (1e-2 if dtype == torch.bfloat16 else 1e-6)
    assert np.all(g64(z)[:, V:] == 0)

