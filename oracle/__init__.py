"""ctypes loader for the float64 CPU oracle (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
may import this package. The product library never loads it.
"""
from __future__ import annotations

import ctypes as ct
import math
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gpt2_oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")

_dp = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_fp = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")
_ip = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_lp = np.ctypeslib.ndpointer(dtype=np.int64, flags="C_CONTIGUOUS")


def build(force: bool = False) -> str:
    """Compile the oracle with g++ (OpenMP, -O2) into oracle/liboracle.so."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["g++", "-O2", "-std=c++17", "-fopenmp", "-fPIC", "-shared", _SRC, "-o", _LIB + ".tmp"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ct.CDLL(build())
        cfgp = ct.POINTER(ct.c_int)
        L.orc_num_params.argtypes = [cfgp]
        L.orc_num_params.restype = ct.c_int64
        L.orc_num_tensors.argtypes = [cfgp]
        L.orc_tensor_info.argtypes = [cfgp, ct.c_int, ct.c_char_p, ct.c_int, ct.POINTER(ct.c_int64),
                                      ct.POINTER(ct.c_int64), ct.POINTER(ct.c_int), ct.POINTER(ct.c_int64),
                                      ct.POINTER(ct.c_int)]
        L.orc_init_params.argtypes = [cfgp, ct.c_uint64, _fp]
        L.orc_init_params.restype = None
        L.orc_forward.argtypes = [cfgp, _dp, _ip, _ip, ct.c_int, ct.c_int, ct.c_int, ct.c_void_p]
        L.orc_forward.restype = ct.c_double
        L.orc_forward_backward.argtypes = [cfgp, _dp, _ip, _ip, ct.c_int, ct.c_int, _dp]
        L.orc_forward_backward.restype = ct.c_double
        L.orc_adamw_step.argtypes = [cfgp, _dp, _dp, _dp, _dp, ct.c_int, ct.c_double, ct.c_double, ct.c_double,
                                     ct.c_double, ct.POINTER(ct.c_double), ct.c_void_p]
        L.orc_adamw_step.restype = None
        L.orc_layernorm_fwd.argtypes = [_dp, _dp, _dp, ct.c_int64, ct.c_int, _dp, _dp, _dp]
        L.orc_layernorm_bwd.argtypes = [_dp, _dp, _dp, _dp, _dp, ct.c_int64, ct.c_int, _dp, _dp, _dp]
        L.orc_linear_fwd.argtypes = [_dp, _dp, ct.c_void_p, ct.c_int64, ct.c_int, ct.c_int, _dp]
        L.orc_linear_bwd.argtypes = [_dp, _dp, _dp, ct.c_int64, ct.c_int, ct.c_int, _dp, _dp, ct.c_void_p]
        L.orc_gelu_fwd.argtypes = [_dp, ct.c_int64, _dp]
        L.orc_gelu_bwd.argtypes = [_dp, _dp, ct.c_int64, _dp]
        L.orc_attention_fwd.argtypes = [_dp, ct.c_int, ct.c_int, ct.c_int, ct.c_int, ct.c_int, _dp, ct.c_void_p]
        L.orc_attention_bwd.argtypes = [_dp, _dp, ct.c_int, ct.c_int, ct.c_int, ct.c_int, _dp]
        L.orc_cross_entropy.argtypes = [_dp, ct.c_int64, ct.c_int, ct.c_int64, _ip, ct.c_double, ct.c_void_p,
                                        ct.c_void_p]
        L.orc_cross_entropy.restype = ct.c_double
        L.orc_token_buckets.argtypes = [_ip, ct.c_int64, ct.c_int, _lp, _lp, _ip]
        L.orc_embedding_bwd.argtypes = [_ip, _dp, ct.c_int, ct.c_int, ct.c_int, _dp, _dp]
        L.orc_embedding_fwd.argtypes = [_ip, _dp, _dp, ct.c_int, ct.c_int, ct.c_int, _dp]
        for f in ("orc_layernorm_fwd", "orc_layernorm_bwd", "orc_linear_fwd", "orc_linear_bwd", "orc_gelu_fwd",
                  "orc_gelu_bwd", "orc_attention_fwd", "orc_attention_bwd", "orc_token_buckets",
                  "orc_embedding_bwd", "orc_embedding_fwd"):
            getattr(L, f).restype = None
        L.orc_set_threads.argtypes = [ct.c_int]
        L.orc_get_threads.restype = ct.c_int
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ct.c_void_p)


@dataclass(frozen=True)
class Config:
    """Model shape: L layers, H heads, width C, context T, logical vocabulary V."""
    L: int
    H: int
    C: int
    T: int
    V: int
    tied: int = 1
    qkv_bias: int = 1

    def arr(self):
        a = (ct.c_int * 7)(self.L, self.H, self.C, self.T, self.V, self.tied, self.qkv_bias)
        return a


@dataclass(frozen=True)
class TensorInfo:
    name: str
    shape: tuple
    offset: int
    decay: bool

    @property
    def size(self) -> int:
        return int(np.prod(self.shape))


def num_params(cfg: Config) -> int:
    return int(lib().orc_num_params(cfg.arr()))


def tensors(cfg: Config) -> list[TensorInfo]:
    L = lib()
    out = []
    name = ct.create_string_buffer(64)
    r, c, o = ct.c_int64(), ct.c_int64(), ct.c_int64()
    nd, dec = ct.c_int(), ct.c_int()
    for i in range(L.orc_num_tensors(cfg.arr())):
        L.orc_tensor_info(cfg.arr(), i, name, 64, ct.byref(r), ct.byref(c), ct.byref(nd), ct.byref(o),
                          ct.byref(dec))
        shape = (r.value, c.value) if nd.value == 2 else (r.value,)
        out.append(TensorInfo(name.value.decode(), shape, o.value, bool(dec.value)))
    return out


def init_params(cfg: Config, seed: int) -> np.ndarray:
    out = np.zeros(num_params(cfg), np.float32)
    lib().orc_init_params(cfg.arr(), seed, out)
    return out


def forward(cfg: Config, params, tokens, targets, attn_mode: int = 0, want_logits: bool = False):
    """Mean cross-entropy (and the logits). attn_mode 0: explicit masked softmax, the
    definition; 1: blocked online softmax, kept for the check that the two agree."""
    p = np.ascontiguousarray(params, np.float64)
    tok = np.ascontiguousarray(tokens, np.int32)
    tgt = np.ascontiguousarray(targets, np.int32)
    B, T = tok.shape
    logits = np.zeros((B * T, cfg.V), np.float64) if want_logits else None
    loss = lib().orc_forward(cfg.arr(), p, tok, tgt, B, T, attn_mode, _ptr(logits))
    return (loss, logits) if want_logits else loss


def forward_backward(cfg: Config, params, tokens, targets):
    p = np.ascontiguousarray(params, np.float64)
    tok = np.ascontiguousarray(tokens, np.int32)
    tgt = np.ascontiguousarray(targets, np.int32)
    B, T = tok.shape
    g = np.zeros_like(p)
    loss = lib().orc_forward_backward(cfg.arr(), p, tok, tgt, B, T, g)
    return loss, g


def adamw_step(cfg: Config, params, grads, m, v, t: int, lr: float, wd: float, b1: float = 0.9,
               b2: float = 0.95, want_clipped: bool = False):
    """In-place AdamW on float64 copies; returns (params, m, v, grad_norm[, clipped])."""
    p = np.array(params, np.float64)
    m = np.array(m, np.float64)
    v = np.array(v, np.float64)
    g = np.ascontiguousarray(grads, np.float64)
    gn = ct.c_double()
    clipped = np.zeros_like(g) if want_clipped else None
    lib().orc_adamw_step(cfg.arr(), p, g, m, v, t, lr, wd, b1, b2, ct.byref(gn), _ptr(clipped))
    return (p, m, v, gn.value, clipped) if want_clipped else (p, m, v, gn.value)


def layernorm_fwd(x, g, b):
    x = np.ascontiguousarray(x, np.float64)
    N, C = x.shape
    y = np.zeros_like(x)
    mean = np.zeros(N)
    rstd = np.zeros(N)
    lib().orc_layernorm_fwd(x, np.ascontiguousarray(g, np.float64), np.ascontiguousarray(b, np.float64), N, C, y,
                            mean, rstd)
    return y, mean, rstd


def layernorm_bwd(dy, x, g, mean, rstd):
    dy = np.ascontiguousarray(dy, np.float64)
    x = np.ascontiguousarray(x, np.float64)
    N, C = x.shape
    dx = np.zeros_like(x)
    dg = np.zeros(C)
    db = np.zeros(C)
    lib().orc_layernorm_bwd(dy, x, np.ascontiguousarray(g, np.float64), np.ascontiguousarray(mean, np.float64),
                            np.ascontiguousarray(rstd, np.float64), N, C, dx, dg, db)
    return dx, dg, db


def linear_fwd(X, W, b=None):
    X = np.ascontiguousarray(X, np.float64)
    W = np.ascontiguousarray(W, np.float64)
    N, K = X.shape
    O = W.shape[0]
    Y = np.zeros((N, O))
    bb = None if b is None else np.ascontiguousarray(b, np.float64)
    lib().orc_linear_fwd(X, W, _ptr(bb), N, K, O, Y)
    return Y


def linear_bwd(dY, X, W):
    dY = np.ascontiguousarray(dY, np.float64)
    X = np.ascontiguousarray(X, np.float64)
    W = np.ascontiguousarray(W, np.float64)
    N, K = X.shape
    O = W.shape[0]
    dX = np.zeros((N, K))
    dW = np.zeros((O, K))
    db = np.zeros(O)
    lib().orc_linear_bwd(dY, X, W, N, K, O, dX, dW, _ptr(db))
    return dX, dW, db


def gelu_fwd(u):
    u = np.ascontiguousarray(u, np.float64)
    a = np.zeros_like(u)
    lib().orc_gelu_fwd(u.ravel(), u.size, a.ravel())
    return a


def gelu_bwd(u, da):
    u = np.ascontiguousarray(u, np.float64)
    da = np.ascontiguousarray(da, np.float64)
    du = np.zeros_like(u)
    lib().orc_gelu_bwd(u.ravel(), da.ravel(), u.size, du.ravel())
    return du


def attention_fwd(qkv, B, T, NH, hd, mode: int = 0):
    qkv = np.ascontiguousarray(qkv, np.float64)
    out = np.zeros((B * T, NH * hd))
    lse = np.zeros((B, NH, T))
    lib().orc_attention_fwd(qkv, B, T, NH, hd, mode, out, _ptr(lse))
    return out, lse


def attention_bwd(qkv, dout, B, T, NH, hd):
    qkv = np.ascontiguousarray(qkv, np.float64)
    dout = np.ascontiguousarray(dout, np.float64)
    dqkv = np.zeros_like(qkv)
    lib().orc_attention_bwd(qkv, dout, B, T, NH, hd, dqkv)
    return dqkv


def cross_entropy(logits, V, targets, scale=1.0, want_grad=True):
    logits = np.ascontiguousarray(logits, np.float64)
    N, ld = logits.shape
    tgt = np.ascontiguousarray(targets, np.int32).ravel()
    dl = np.zeros_like(logits) if want_grad else None
    rl = np.zeros(N)
    tot = lib().orc_cross_entropy(logits, N, V, ld, tgt, scale, _ptr(dl), _ptr(rl))
    return tot, rl, dl


def token_buckets(tokens, V):
    tok = np.ascontiguousarray(tokens, np.int32).ravel()
    counts = np.zeros(V, np.int64)
    offsets = np.zeros(V, np.int64)
    pos = np.zeros(tok.size, np.int32)
    lib().orc_token_buckets(tok, tok.size, V, counts, offsets, pos)
    return counts, offsets, pos


def embedding_fwd(tokens, wte, wpe):
    tok = np.ascontiguousarray(tokens, np.int32)
    B, T = tok.shape
    C = wte.shape[1]
    x0 = np.zeros((B * T, C))
    lib().orc_embedding_fwd(tok, np.ascontiguousarray(wte, np.float64), np.ascontiguousarray(wpe, np.float64), B, T,
                            C, x0)
    return x0


def embedding_bwd(tokens, dx0, V, Tmax=None):
    tok = np.ascontiguousarray(tokens, np.int32)
    B, T = tok.shape
    dx0 = np.ascontiguousarray(dx0, np.float64)
    C = dx0.shape[1]
    dwte = np.zeros((V, C))
    dwpe = np.zeros((Tmax or T, C))
    lib().orc_embedding_bwd(tok, dx0, B, T, C, dwte, dwpe)
    return dwte, dwpe


def set_threads(n: int) -> None:
    lib().orc_set_threads(n)


def get_threads() -> int:
    return int(lib().orc_get_threads())


def lr_schedule(step: int, max_lr: float = 6e-4, min_lr: float = 6e-5, warmup: int = 715,
                total: int = 19073) -> float:
    """Learning rate at optimizer step `step` (0-based), in float64.

    "AxonLM", Training Recipe table: peak 6e-4, minimum 6e-5 (peak / 10), 715 warmup steps,
    19,073 total steps; "AxonLM", Key Features, and "Genesis", Training Features: linear
    warmup, then cosine decay. Reading (the pages leave the indexing open): warmup step s takes
    peak * (s + 1) / warmup; from s = warmup the rate is
    min + (peak - min) * (1 + cos(pi * (s - warmup) / (total - warmup))) / 2, reaching the
    minimum at s = total and staying there.
    """
    if step < warmup:
        return max_lr * float(step + 1) / float(warmup)
    if step >= total:
        return min_lr
    x = math.pi * float(step - warmup) / float(total - warmup)
    return min_lr + (max_lr - min_lr) * (1.0 + math.cos(x)) / 2.0


def sample_topk(z, k: int, temperature: float, top_p: float, u: float) -> int:
    """Index drawn from one logits row by temperature / top-k / top-p sampling.

    "GPT From Scratch", Architecture diagram: generation samples with temperature and
    top-k; "Genesis", Project Structure and What I built from scratch: temperature, top-k
    and top-p (nucleus) sampling. The pages give no tie or precision rule; the reading:
    rank the logits by value, larger first, equal values by lower index (-0.0 equals
    +0.0); keep the first k; weight each kept logit by exp((z - z_max) / temperature) in
    float64; form running sums c_0, c_1, ... of the weights in rank order; with top_p < 1
    keep only ranks up to the first one whose running sum reaches top_p * c_{k-1}; return
    the first kept rank whose running sum exceeds u * (running sum of the last kept rank),
    or the last kept rank. temperature and top_p are taken at float32 precision (the
    library's argument type), u in float64.
    """
    z = [float(x) for x in np.asarray(z, dtype=np.float32).reshape(-1)]
    V = len(z)
    if not (1 <= k <= V):
        raise ValueError("1 <= k <= V")
    temperature = float(np.float32(temperature))
    top_p = float(np.float32(top_p))
    ranked = sorted(range(V), key=lambda i: (-z[i], i))[:k]
    zmax = z[ranked[0]]
    weights = [math.exp((z[i] - zmax) / temperature) for i in ranked]
    running = []
    acc = 0.0
    for w in weights:
        acc += w
        running.append(acc)
    last = k - 1
    if top_p < 1.0:
        for j in range(k):
            if running[j] >= top_p * running[k - 1]:
                last = j
                break
    target = u * running[last]
    for j in range(last + 1):
        if running[j] > target:
            return ranked[j]
    return ranked[last]
