"""Time one kernel of the library at a chosen shape with CUDA events.

    python -m train_step_b200.kernel_bench gemm --M 16384 --N 3072 --K 768 --epi 1
    python -m train_step_b200.kernel_bench attn --B 16 --T 1024 --H 12
    python -m train_step_b200.kernel_bench ln --N 16384 --C 768

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


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("kernel", choices=["gemm", "attn", "attn_bwd", "ln", "ce"])
    ap.add_argument("--M", type=int, default=16384)
    ap.add_argument("--N", type=int, default=3072)
    ap.add_argument("--K", type=int, default=768)
    ap.add_argument("--epi", type=int, default=0)
    ap.add_argument("--a-mn", action="store_true")
    ap.add_argument("--b-mn", action="store_true")
    ap.add_argument("--ksplit", type=int, default=1, help="0 = the library's choice")
    ap.add_argument("--bn", type=int, default=0, help="GEMM tile width: 0 = the library's choice, 128 or 256")
    ap.add_argument("--B", type=int, default=16)
    ap.add_argument("--T", type=int, default=1024)
    ap.add_argument("--H", type=int, default=12)
    ap.add_argument("--C", type=int, default=768)
    ap.add_argument("--V", type=int, default=50257)
    ap.add_argument("--iters", type=int, default=20)
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
                            ld_aux=N, ksplit=a.ksplit, bn=a.bn, iters=a.iters)
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
