"""Time one kernel of the library at a chosen shape with CUDA events.

    python -m train_step_b200.kernel_bench gemm --M 16384 --N 3072 --K 768 --epi 1
    python -m train_step_b200.kernel_bench attn --B 16 --T 1024 --H 12
    python -m train_step_b200.kernel_bench ln --N 16384 --C 768
    python -m train_step_b200.kernel_bench decode --B 16 --T0 512 --steps 64

Used for focused profiler captures of one kernel on a small case. Inputs are
seeded random tensors; nothing is checked here (the tests check numerics).
"""
from __future__ import annotations

import argparse
import json

import torch

import train_step_b200 as tsb


def timeit(fn, iters: int, warmup: int = 3) -> float:
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(iters):
        fn()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / iters


def hbm_peak():
    """(GB/s, 'measured' | 'fallback'): the copy bandwidth measured on this GPU type."""
    import os
    path = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def gemv_bench(a) -> dict:
    """The generation step's skinny products (GPT-2 124M shapes) timed alone: `iters`
    back-to-back launches, plain and as programmatic dependents. One weight matrix is
    reused, so after the first launch it is served from L2: this is each kernel's latency
    floor, not its HBM-bound time."""
    C, V = a.C, a.V
    shapes = {"qkv+ln": (3 * C, C, 0, True), "attn_out": (C, C, 2, False), "fc+ln": (4 * C, C, 1, True),
              "proj": (C, 4 * C, 2, False), "head+ln": (V, C, 4, True)}
    out = {}
    for name, (N, K, epi, ln) in shapes.items():
        B = a.B
        x = torch.randn(B, K, device="cuda", dtype=torch.float32 if ln else torch.bfloat16)
        W = torch.randn(N, K, device="cuda").to(torch.bfloat16)
        bias = torch.zeros(N, device="cuda")
        g = torch.ones(K, device="cuda") if ln else None
        b = torch.zeros(K, device="cuda") if ln else None
        resid = torch.zeros(B, N, device="cuda") if epi == 2 else None
        o = torch.empty(B, N, device="cuda", dtype=torch.float32 if epi in (2, 4) else torch.bfloat16)
        row = {}
        for pdl in (False, True):
            ms = tsb.gemv(x, W, o, B=B, N=N, K=K, epilogue=epi, bias=bias, resid=resid, ldr=N, ln_g=g, ln_b=b,
                          iters=a.iters, pdl=pdl)
            row["pdl" if pdl else "plain"] = dict(us=ms * 1e3, gbs=2.0 * N * K / (ms * 1e-3) / 1e9)
        out[name] = row
    return dict(B=a.B, gemv=out)


def decode_bench(a) -> dict:
    """Generation with the key/value cache on GPT-2 124M (random weights): B prompts of T0
    tokens, then `steps` decode steps, each one forward step for all B sequences followed
    by the sampler. Reports milliseconds per decode step (forward + sampling), generated
    tokens per second, and the step's algorithmic HBM bytes over its time against the
    measured copy bandwidth: every bf16 weight once, the fp32 LayerNorm parameters and
    biases, the cache rows read (positions 0..p of every layer and sequence) and written."""
    import numpy as np
    cfg = tsb.Config(L=12, H=a.H, C=a.C, T=1024, V=a.V, tied=1, qkv_bias=1, dtype=tsb.BF16, B_max=a.B)
    stream = torch.cuda.Stream()
    torch.cuda.set_stream(stream)
    m = tsb.GPT2(cfg, seed=1, stream=stream.cuda_stream)
    B, T0, steps = a.B, a.T0, a.steps
    if T0 + steps > cfg.T:
        raise SystemExit("T0 + steps must not exceed 1024")
    prompt = torch.randint(0, cfg.V, (B, T0), dtype=torch.int32, device="cuda")
    u = torch.from_numpy(np.random.default_rng(0).random((steps, B))).cuda()
    idx = torch.empty(B, dtype=torch.int32, device="cuda")
    logits = torch.empty(B, cfg.V, dtype=torch.float32, device="cuda")

    def run(n):
        m.prefill(prompt, logits_out=logits)
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for s in range(n):
            m.sample_topk(logits, a.topk, 1.0, 1.0, u[s], out=idx, sync=False)
            m.decode_step(idx, logits_out=logits, sync=False)
        t1.record(stream)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1) / n

    run(min(steps, 8))
    ms = run(steps)
    n0 = m.launch_count()
    run(steps)
    launches = (m.launch_count() - n0) / steps  # includes the prefill's launches, spread over the steps
    m.profile(True)
    run(steps)
    prof = {k: dict(ms_per_step=v[0] / steps, launches_per_step=v[1] / steps, gbs=v[3] / (v[0] * 1e-3) / 1e9)
            for k, v in m.profile_read().items() if v[1] > 0 and k.startswith(("decode", "sample", "layernorm_fwd",
                                                                               "embedding_fwd"))}
    m.profile(False)
    L, C, V = cfg.L, cfg.C, cfg.V
    F = 4 * C
    w_bytes = 2.0 * (L * (3 * C * C + C * C + 2 * F * C) + V * C)
    p_bytes = 4.0 * (L * (3 * C + C + F + C + 4 * C) + 2 * C)
    mean_pos = T0 + (steps - 1) / 2.0
    kv_bytes = 2.0 * L * B * 2 * C * (mean_pos + 1) + 2.0 * L * B * 2 * C
    step_bytes = w_bytes + p_bytes + kv_bytes
    gbs = step_bytes / (ms * 1e-3) / 1e9
    return dict(shape=[B, T0, steps], ms_per_step=ms, tokens_per_s=B / (ms * 1e-3), bytes_per_step=step_bytes,
                gbs=gbs, hbm_frac=gbs / hbm_peak()[0], peak_kind=hbm_peak()[1], launches_per_step=launches,
                kernels=prof)


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("kernel", choices=["gemm", "attn", "attn_bwd", "ln", "ln_bwd", "ce", "decode", "gemv"])
    ap.add_argument("--M", type=int, default=16384)
    ap.add_argument("--N", type=int, default=3072)
    ap.add_argument("--K", type=int, default=768)
    ap.add_argument("--epi", type=int, default=0)
    ap.add_argument("--a-mn", action="store_true")
    ap.add_argument("--b-mn", action="store_true")
    ap.add_argument("--ksplit", type=int, default=1, help="0 = the library's choice")
    ap.add_argument("--bn", type=int, default=0, help="GEMM tile width: 0 = the library's choice, 128 or 256")
    ap.add_argument("--pair", type=int, default=-1, help="GEMM 2-CTA tiles: -1 = the library's choice, 0 off, 1 on")
    ap.add_argument("--B", type=int, default=16)
    ap.add_argument("--T", type=int, default=1024)
    ap.add_argument("--H", type=int, default=12)
    ap.add_argument("--C", type=int, default=768)
    ap.add_argument("--V", type=int, default=50257)
    ap.add_argument("--iters", type=int, default=20)
    ap.add_argument("--stored", action="store_true", help="attn_bwd: the training step's stored-dS form")
    ap.add_argument("--T0", type=int, default=512, help="decode: prompt length")
    ap.add_argument("--steps", type=int, default=64, help="decode: generated tokens per sequence")
    ap.add_argument("--topk", type=int, default=50, help="decode: k of the sampler")
    a = ap.parse_args()
    g = torch.Generator(device="cuda").manual_seed(0)
    dev = "cuda"
    res = {"kernel": a.kernel}
    if a.kernel == "gemm":
        M, N, K = a.M, a.N, a.K
        A = torch.randn((K, M) if a.a_mn else (M, K), device=dev, generator=g).to(torch.bfloat16)
        B = torch.randn((K, N) if a.b_mn else (N, K), device=dev, generator=g).to(torch.bfloat16)
        f32 = a.epi in (2, 4)
        out = torch.zeros(M, N, device=dev, dtype=torch.float32 if f32 else torch.bfloat16)
        out2 = torch.zeros(M, N, device=dev, dtype=torch.bfloat16) if a.epi == 1 else None
        bias = torch.zeros(N, device=dev) if a.epi in (0, 1, 2) else None
        aux = None
        if a.epi == 2:
            aux = torch.zeros(M, N, device=dev)
        elif a.epi == 3:
            aux = torch.zeros(M, N, device=dev, dtype=torch.bfloat16)

        ms = tsb.gemm_bench(A, B, out, M=M, N=N, K=K, lda=M if a.a_mn else K, ldb=N if a.b_mn else K, ldo=N,
                            a_mn=a.a_mn, b_mn=a.b_mn, epilogue=a.epi, out2=out2, ldo2=N, bias=bias, aux=aux,
                            ld_aux=N, ksplit=a.ksplit, bn=a.bn, pair=a.pair, iters=a.iters)
        res.update(shape=[M, N, K], ms=ms, tflops=2.0 * M * N * K / (ms * 1e-3) / 1e12)
    elif a.kernel in ("attn", "attn_bwd"):
        B, T, H, hd = a.B, a.T, a.H, 64
        C = H * hd
        qkv = torch.randn(B * T, 3 * C, device=dev, generator=g).to(torch.bfloat16)
        out = torch.zeros(B * T, C, device=dev, dtype=torch.bfloat16)
        lse = torch.zeros(B, H, T, device=dev)
        tsb.attention_fwd(qkv, out, lse, B, T, H, hd)
        dout = torch.randn(B * T, C, device=dev, generator=g).to(torch.bfloat16)
        dqkv = torch.zeros_like(qkv)
        if a.kernel == "attn":
            ms = timeit(lambda: tsb.attention_fwd(qkv, out, lse, B, T, H, hd), a.iters)
            fl = 4.0 * B * H * hd * T * (T + 1) / 2
        elif a.stored:
            ds = torch.empty(tsb.attention_ds_bytes(B, T, H) // 2, dtype=torch.bfloat16, device=dev)
            ms = timeit(lambda: tsb.attention_bwd_stored(qkv, out, dout, lse, dqkv, ds, B, T, H, hd), a.iters)
            fl = 2.5 * 4.0 * B * H * hd * T * (T + 1) / 2
        else:
            ms = timeit(lambda: tsb.attention_bwd(qkv, out, dout, lse, dqkv, B, T, H, hd), a.iters)
            fl = 2.5 * 4.0 * B * H * hd * T * (T + 1) / 2
        res.update(shape=[B, T, H, hd], ms=ms, tflops=fl / (ms * 1e-3) / 1e12)
    elif a.kernel == "ln":
        N, C = a.M, a.C
        x = torch.randn(N, C, device=dev, generator=g)
        w = torch.ones(C, device=dev)
        bb = torch.zeros(C, device=dev)
        y = torch.zeros(N, C, device=dev, dtype=torch.bfloat16)
        mean = torch.zeros(N, device=dev)
        rstd = torch.zeros(N, device=dev)
        ms = timeit(lambda: tsb.layernorm_fwd(x, w, bb, y, mean, rstd), a.iters)
        res.update(shape=[N, C], ms=ms, gbs=N * C * 6 / (ms * 1e-3) / 1e9)
    elif a.kernel == "ln_bwd":
        N, C = a.M, a.C
        x = torch.randn(N, C, device=dev, generator=g)
        w = torch.ones(C, device=dev)
        bb = torch.zeros(C, device=dev)
        y = torch.zeros(N, C, device=dev, dtype=torch.bfloat16)
        mean = torch.zeros(N, device=dev)
        rstd = torch.zeros(N, device=dev)
        tsb.layernorm_fwd(x, w, bb, y, mean, rstd)
        dy = torch.randn(N, C, device=dev, generator=g)
        dres = torch.randn(N, C, device=dev, generator=g)
        dres_act = torch.zeros(N, C, device=dev, dtype=torch.bfloat16)
        dg = torch.zeros(C, device=dev)
        db = torch.zeros(C, device=dev)
        ms = timeit(lambda: tsb.layernorm_bwd(dy, x, w, mean, rstd, dres, dres_act, dg, db, accumulate=True,
                                              accumulate_params=True), a.iters)
        res.update(shape=[N, C], ms=ms, gbs=N * C * 18 / (ms * 1e-3) / 1e9)
    elif a.kernel == "decode":
        res.update(decode_bench(a))
    elif a.kernel == "gemv":
        res.update(gemv_bench(a))
    else:
        N, V = a.M, a.V
        ld = (V + 63) // 64 * 64
        z = torch.randn(N, ld, device=dev, generator=g).to(torch.bfloat16)
        tgt = torch.randint(0, V, (N,), device=dev, generator=g, dtype=torch.int32)
        rl = torch.zeros(N, device=dev)
        ms = timeit(lambda: tsb.cross_entropy(z, V, tgt, 1.0 / N, rl), a.iters)
        res.update(shape=[N, ld], ms=ms, gbs=2 * N * ld * 2 / (ms * 1e-3) / 1e9)
    print(json.dumps(res))


if __name__ == "__main__":
    main()
