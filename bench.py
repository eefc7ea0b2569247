#!/usr/bin/env python
"""Training throughput of the GPT-2 pre-LN step on B200: tokens/s and MFU.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config gpt2-124m] [--impl ours|reference]

One step = `accum` micro-batches of forward + backward (gradient accumulation)
followed by one global-norm-clipped AdamW update, on seeded synthetic Zipf(1.1)
tokens (stand-in for the pages' BPE text corpora). For N > 1 (torchrun, one
process per GPU) every rank runs its own micro-batches (weak scaling) and the
gradients are averaged with NCCL all-reduces, one per layer bucket, that overlap the
last micro-batch's backward pass (data parallel).

Prints one JSON line (rank 0). `value` is whole-job tokens/s with the inputs
already resident in HBM; `e2e` is the same metric through the public C-ABI with
token buffers in pinned host memory, copied in each step, and the loss and grad
norm read back each step. MFU counts 6 N_params + 12 L T C FLOPs per token.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "train tokens/sec and MFU, GPT-2 124M, T=1024 bf16, 1×B200"
PAGES_L4_TOKENS_PER_S = 40000.0  # "slimgpt": ~40k tokens/s, GPT-2 124M bf16 on one NVIDIA L4 (context)

CONFIGS = {
    "gpt2-124m": dict(L=12, H=12, C=768, T=1024, V=50257, tied=1, qkv_bias=1, B=16, accum=4),
    "gpt2-124m-untied": dict(L=12, H=12, C=768, T=1024, V=50257, tied=0, qkv_bias=0, B=32, accum=1),
    "gpt2-355m": dict(L=24, H=16, C=1024, T=1024, V=50257, tied=1, qkv_bias=1, B=8, accum=8),
    "gpt2-1558m": dict(L=48, H=25, C=1600, T=1024, V=50257, tied=1, qkv_bias=1, B=4, accum=1),
}
LR, WD, B1, B2 = 6e-4, 0.1, 0.9, 0.95


def n_params(c) -> int:
    C, L, V, T = c["C"], c["L"], c["V"], c["T"]
    per = 2 * C + 3 * C * C + (3 * C if c["qkv_bias"] else 0) + C * C + C + 2 * C + 4 * C * C + 4 * C + 4 * C * C + C
    return V * C + T * C + L * per + 2 * C + (0 if c["tied"] else V * C)


def flops_per_token(c) -> float:
    return 6.0 * n_params(c) + 12.0 * c["L"] * c["T"] * c["C"]


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms in the background."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        self.gpu = gpu_index
        self.path = os.path.join("/tmp", f"bench_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", str(self.gpu)], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    d = os.path.join(ROOT, "train_step_b200", "csrc")
    for f in sorted(os.listdir(d)):
        h.update(open(os.path.join(d, f), "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str):
    """Per-launch DRAM bytes of `kernel` from the committed ncu summary, if it
    was taken from the current kernel sources; else None."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    e = d.get(kernel)
    if not e or e.get("source_hash") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


def cpu_baseline(c, seconds_hint=True):
    """The float64 oracle, as it stands, on a bounded sample of the same workload:
    one sequence of T=256 tokens of the same model shape, forward + backward, then
    one AdamW step over all parameters."""
    import oracle
    from train_step_b200 import synth
    oc = oracle.Config(c["L"], c["H"], c["C"], c["T"], c["V"], c["tied"], c["qkv_bias"])
    p = oracle.init_params(oc, 42).astype(np.float64)
    Ts = 256
    tok, tgt = synth.micro_batch(1, Ts, c["V"])
    t0 = time.perf_counter()
    _, g = oracle.forward_backward(oc, p, tok, tgt)
    oracle.adamw_step(oc, p, g, np.zeros_like(p), np.zeros_like(p), 1, LR, WD, B1, B2)
    dt = time.perf_counter() - t0
    out = {"value": Ts / dt, "unit": "tokens/s", "cores": oracle.get_threads(), "kind": "oracle",
           "sample": f"1 sequence x {Ts} tokens of the {c['L']}-layer C={c['C']} model: float64 forward+backward "
                     f"and one AdamW step ({dt:.1f} s)"}
    # the same on one thread (a shorter sample), and the tiny character-level config's full step
    threads = oracle.get_threads()
    T1 = 32
    tok1, tgt1 = synth.micro_batch(1, T1, c["V"], index=1)
    oracle.set_threads(1)
    try:
        t0 = time.perf_counter()
        _, g = oracle.forward_backward(oc, p, tok1, tgt1)
        oracle.adamw_step(oc, p, g, np.zeros_like(p), np.zeros_like(p), 1, LR, WD, B1, B2)
        dt1 = time.perf_counter() - t0
    finally:
        oracle.set_threads(threads)
    out["single_thread"] = {"value": T1 / dt1, "unit": "tokens/s", "cores": 1,
                            "sample": f"1 sequence x {T1} tokens, same model and work ({dt1:.1f} s)"}
    tc = oracle.Config(4, 4, 128, 64, 65, 1, 1)
    tp = oracle.init_params(tc, 42).astype(np.float64)
    ttok, ttgt = synth.micro_batch(8, 64, 65, dist="uniform")
    t0 = time.perf_counter()
    _, g = oracle.forward_backward(tc, tp, ttok, ttgt)
    oracle.adamw_step(tc, tp, g, np.zeros_like(tp), np.zeros_like(tp), 1, LR, WD, B1, B2)
    dtt = time.perf_counter() - t0
    out["tiny_step"] = {"value": 8 * 64 / dtt, "unit": "tokens/s", "cores": threads,
                        "sample": f"tiny config (L4 H4 C128 T64 V65), B=8: one full step ({dtt * 1e3:.1f} ms)"}
    return out


def run_reference(args, c):
    """The oracle as the reference arm: each step is a bounded sample (one
    sequence of 64 tokens, forward + backward + AdamW), on the host cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    from train_step_b200 import synth
    oc = oracle.Config(c["L"], c["H"], c["C"], c["T"], c["V"], c["tied"], c["qkv_bias"])
    p = oracle.init_params(oc, 42).astype(np.float64)
    m = np.zeros_like(p)
    v = np.zeros_like(p)
    Ts = 64
    times = []
    for s in range(args.warmup + args.steps):
        tok, tgt = synth.micro_batch(1, Ts, c["V"], index=s)
        t0 = time.perf_counter()
        _, g = oracle.forward_backward(oc, p, tok, tgt)
        p, m, v, _ = oracle.adamw_step(oc, p, g, m, v, s + 1, LR, WD, B1, B2)
        times.append(time.perf_counter() - t0)
    dt = float(np.mean(times[args.warmup:]))
    value = Ts / dt
    sample = f"1 sequence x {Ts} tokens per step, float64 forward+backward+AdamW on {oracle.get_threads()} threads"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic Zipf(1.1) tokens",
            "config": {"workload": args.config, "sample_tokens_per_step": Ts},
            "mfu": value * flops_per_token(c) / 2.25e15,
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.get_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default="gpt2-124m", choices=sorted(CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-steps", type=int, default=2)
    args = ap.parse_args()
    c = CONFIGS[args.config]
    if args.impl == "reference":
        return run_reference(args, c)

    import torch
    import train_step_b200 as tsb
    from train_step_b200 import dp, synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")

    B, T, accum = c["B"], c["T"], c["accum"]
    cfg = tsb.Config(L=c["L"], H=c["H"], C=c["C"], T=T, V=c["V"], tied=c["tied"], qkv_bias=c["qkv_bias"],
                     dtype=tsb.BF16, B_max=B)
    # one dedicated stream for the library's kernels, the token copies and the timing
    # events (torch's default stream has handle 0, which the library does not share)
    stream = torch.cuda.Stream()
    torch.cuda.set_stream(stream)
    model = tsb.GPT2(cfg, seed=42, stream=stream.cuda_stream)

    # inputs resident in HBM: this rank's micro-batches (weak scaling by rank)
    mbs = [synth.micro_batch(B, T, c["V"], index=i) for i in dp.micro_batch_indices(rank, world, accum)]
    dev_in = [(torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda()) for a, b in mbs]

    # data parallel: the gradient average runs bucket by bucket (a layer at a time) on its
    # own stream while the last micro-batch's backward pass is still running
    exchange = dp.BucketedAllReduce(model) if dist is not None else None

    def train_step(inputs, want_outputs=False):
        loss = None
        for j, (tok, tgt) in enumerate(inputs):
            last = j == len(inputs) - 1
            if exchange is not None and last:
                exchange.arm()
            loss = model.forward_backward(tok, tgt, want_loss=want_outputs and last and exchange is None)
        if exchange is not None:
            exchange.run()
            if want_outputs:
                loss = model.read_loss()
        gn = model.step(LR, WD, B1, B2, want_norm=want_outputs)
        return loss, gn

    def barrier():
        if dist is not None:
            dist.barrier()

    for _ in range(args.warmup):
        train_step(dev_in)
    torch.cuda.synchronize()
    barrier()
    clocks = ClockSampler(local)
    clocks.start()
    launches0 = model.launch_count()
    torch.cuda.synchronize()
    barrier()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        train_step(dev_in)
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = ev0.elapsed_time(ev1) / args.steps
    clk = clocks.stop()
    launches = model.launch_count() - launches0
    if dist is not None:
        t = torch.tensor([ms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    tokens_per_step = B * T * accum * world
    value = tokens_per_step / (ms / 1e3)
    fpt = flops_per_token(c)
    peaks, peak_src = measured_peaks()
    mfu_nominal = value * fpt / (2.25e15 * world)
    mfu_measured = value * fpt / (peaks["bf16_tflops_sustained"] * 1e12 * world)

    # per-kernel breakdown with CUDA events on the library's stream (separate steps)
    model.profile(True)
    for _ in range(args.profile_steps):
        train_step(dev_in)
    model.profile(False)
    prof = model.profile_read()
    torch.cuda.synchronize()
    kernels = {}
    for name, (kms, n, fl, by) in prof.items():
        if n == 0:
            continue
        per = kms / args.profile_steps
        kernels[name] = {"ms_per_step": round(per, 4), "launches_per_step": n // args.profile_steps,
                         "share": None}
        if fl > 0:
            kernels[name]["tflops"] = round(fl / (kms * 1e-3) / 1e12, 1)
        if by > 0:
            kernels[name]["gbs"] = round(by / (kms * 1e-3) / 1e9, 1)
    if not kernels:
        raise SystemExit("--profile-steps must be >= 1 (the roofline needs per-kernel times)")
    tot = sum(k["ms_per_step"] for k in kernels.values()) or 1.0
    for k in kernels.values():
        k["share"] = round(k["ms_per_step"] / tot, 4)
    # the tensor-core GEMM is one kernel, profiled by role (forward, head, dX, dW)
    gemm_roles = [k for k in prof if k.startswith("gemm_tc")]
    prof_agg = dict(prof)
    if gemm_roles:
        prof_agg["gemm_tc"] = tuple(sum(prof[k][i] for k in gemm_roles) for i in range(4))
        for k in gemm_roles:
            prof_agg.pop(k)
    dom = max(prof_agg, key=lambda k: prof_agg[k][0])
    dms, dn, dfl, dby = prof_agg[dom]
    if dfl > 0:
        achieved = dfl / (dms * 1e-3) / 1e12
        peak = peaks["bf16_tflops_sustained"]
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
                "frac": round(achieved / peak, 4), "kernel": dom,
                "peak_source": f"{peak_src} cuBLAS bf16, sustained (timed inside a long step)"}
    else:
        achieved = dby / (dms * 1e-3) / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "kernel": dom, "peak_source": f"{peak_src} copy bandwidth"}
    tr = ncu_traffic(dom)
    roof["traffic"] = tr
    roof["launches_per_step"] = dn // args.profile_steps

    # end to end through the public API with host (pinned) token buffers
    e2e = None
    if not args.no_e2e:
        host_in = []
        for a, b in mbs:
            ta = torch.from_numpy(a).pin_memory()
            tb = torch.from_numpy(b).pin_memory()
            host_in.append((ta, tb))
        for _ in range(2):
            train_step(host_in, want_outputs=True)
        torch.cuda.synchronize()
        barrier()
        t0 = time.perf_counter()
        for _ in range(args.steps):
            loss, gn = train_step(host_in, want_outputs=True)
        torch.cuda.synchronize()
        barrier()
        e2e_s = (time.perf_counter() - t0) / args.steps
        if dist is not None:
            t = torch.tensor([e2e_s], device="cuda")
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            e2e_s = float(t.item())
        e2e = {"value": tokens_per_step / e2e_s, "unit": "tokens/s",
               "h2d_bytes_per_step": int(sum(a.numel() * 4 + b.numel() * 4 for a, b in host_in)),
               "d2h_bytes_per_step": 8, "loss": loss, "grad_norm": gn}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(c)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": value / PAGES_L4_TOKENS_PER_S,
            "dtype": "bf16", "data": "synthetic Zipf(1.1) token ids over [0, 50257), seeded (splitmix64)",
            "config": {"workload": args.config, "global_batch": B * accum * world, "micro_batch": B,
                       "grad_accum": accum, "seq_len": T, "parallelism": f"dp{world}",
                       "tokens_per_step": tokens_per_step, "l2": "inputs larger than L2 (activations ~5 GB)"},
            "mfu": mfu_nominal, "mfu_vs_measured_sustained_peak": mfu_measured,
            "flops_per_token": fpt, "n_params": n_params(c),
            "roofline": roof, "kernels": kernels, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": launches, "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    model.close()
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
