"""Python binding of the B200 GPT-2 training-step library (include/gpt2.h).

Argument marshalling only: every step of the training step runs in the CUDA
kernels of ``libgpt2_b200.so``. PyTorch supplies device memory and streams. If
the shared library is missing this module raises; there is no fallback.
"""
from __future__ import annotations

import ctypes as ct
import os
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgpt2_b200.so")

FP32, BF16 = 0, 1
EPI_BIAS, EPI_BIAS_GELU, EPI_RESID, EPI_DGELU, EPI_F32 = 0, 1, 2, 3, 4

ERRORS = {
    -1: "GPT2_ERR_CONFIG", -2: "GPT2_ERR_OOM", -3: "GPT2_ERR_SEQ_TOO_LONG", -4: "GPT2_ERR_TOKEN_RANGE",
    -5: "GPT2_ERR_BATCH", -6: "GPT2_ERR_NO_GRAD", -7: "GPT2_ERR_CUDA", -8: "GPT2_ERR_TIMEOUT",
}


class Gpt2Error(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{ERRORS.get(code, code)}: {msg}")
        self.code = code


class _Config(ct.Structure):
    _fields_ = [(n, ct.c_int) for n in ("L", "H", "C", "T", "V", "tied", "qkv_bias", "dtype", "B_max")]


_lib = None
_SYMBOLS = {
    "gpt2_create": ([ct.POINTER(_Config), ct.c_uint64, ct.POINTER(ct.c_void_p)], ct.c_int),
    "gpt2_set_stream": ([ct.c_void_p, ct.c_void_p], ct.c_int),
    "gpt2_forward_backward": ([ct.c_void_p, ct.c_void_p, ct.c_void_p, ct.c_int, ct.c_int, ct.c_void_p], ct.c_int),
    "gpt2_forward": ([ct.c_void_p, ct.c_void_p, ct.c_void_p, ct.c_int, ct.c_int, ct.c_void_p], ct.c_int),
    "gpt2_step": ([ct.c_void_p, ct.c_float, ct.c_float, ct.c_float, ct.c_float, ct.c_void_p], ct.c_int),
    "gpt2_zero_grad": ([ct.c_void_p], ct.c_int),
    "gpt2_num_params": ([ct.c_void_p, ct.POINTER(ct.c_int64)], ct.c_int),
    "gpt2_tensor_info": ([ct.c_void_p, ct.c_int, ct.c_char_p, ct.c_int, ct.POINTER(ct.c_int64),
                          ct.POINTER(ct.c_int64), ct.POINTER(ct.c_int), ct.POINTER(ct.c_int64)], ct.c_int),
    "gpt2_get_params": ([ct.c_void_p, ct.c_void_p, ct.c_int64], ct.c_int),
    "gpt2_set_params": ([ct.c_void_p, ct.c_void_p, ct.c_int64], ct.c_int),
    "gpt2_get_grads": ([ct.c_void_p, ct.c_void_p, ct.c_int64], ct.c_int),
    "gpt2_get_adam": ([ct.c_void_p, ct.c_void_p, ct.c_void_p, ct.c_int64, ct.POINTER(ct.c_int64)], ct.c_int),
    "gpt2_set_adam": ([ct.c_void_p, ct.c_void_p, ct.c_void_p, ct.c_int64, ct.c_int64], ct.c_int),
    "gpt2_launch_count": ([ct.c_void_p, ct.POINTER(ct.c_int64)], ct.c_int),
    "gpt2_grad_buffer": ([ct.c_void_p, ct.POINTER(ct.c_void_p), ct.POINTER(ct.c_int64)], ct.c_int),
    "gpt2_profile": ([ct.c_void_p, ct.c_int], ct.c_int),
    "gpt2_profile_read": ([ct.c_void_p, ct.c_int, ct.c_char_p, ct.c_int, ct.POINTER(ct.c_double),
                           ct.POINTER(ct.c_int64), ct.POINTER(ct.c_double), ct.POINTER(ct.c_double)], ct.c_int),
    "gpt2_last_error": ([ct.c_void_p], ct.c_char_p),
    "gpt2_destroy": ([ct.c_void_p], None),
    "gpt2_op_gemm": ([ct.c_int, ct.c_void_p, ct.c_int64, ct.c_int, ct.c_void_p, ct.c_int64, ct.c_int, ct.c_int,
                      ct.c_int, ct.c_int, ct.c_int, ct.c_void_p, ct.c_int64, ct.c_void_p, ct.c_int64, ct.c_void_p,
                      ct.c_void_p, ct.c_int64, ct.c_int, ct.c_int, ct.c_void_p], ct.c_int),
    "gpt2_op_gemm_bench": ([ct.c_void_p, ct.c_int64, ct.c_int, ct.c_void_p, ct.c_int64, ct.c_int, ct.c_int, ct.c_int,
                            ct.c_int, ct.c_int, ct.c_void_p, ct.c_int64, ct.c_void_p, ct.c_int64, ct.c_void_p,
                            ct.c_void_p, ct.c_int64, ct.c_int, ct.c_int, ct.c_int, ct.c_int, ct.c_int,
                            ct.POINTER(ct.c_float), ct.c_void_p], ct.c_int),
    "gpt2_op_layernorm_fwd": ([ct.c_int, ct.c_void_p, ct.c_void_p, ct.c_void_p, ct.c_int, ct.c_int, ct.c_void_p,
                               ct.c_void_p, ct.c_void_p, ct.c_void_p], ct.c_int),
    "gpt2_op_layernorm_bwd": ([ct.c_int, ct.c_void_p, ct.c_void_p, ct.c_void_p, ct.c_void_p, ct.c_void_p, ct.c_int,
                               ct.c_int, ct.c_void_p, ct.c_void_p, ct.c_int, ct.c_void_p, ct.c_void_p, ct.c_int,
                               ct.c_void_p], ct.c_int),
    "gpt2_op_attention_fwd": ([ct.c_int, ct.c_void_p, ct.c_int, ct.c_int, ct.c_int, ct.c_int, ct.c_void_p,
                               ct.c_void_p, ct.c_void_p], ct.c_int),
    "gpt2_op_attention_bwd": ([ct.c_int, ct.c_void_p, ct.c_void_p, ct.c_void_p, ct.c_void_p, ct.c_int, ct.c_int,
                               ct.c_int, ct.c_int, ct.c_void_p, ct.c_void_p], ct.c_int),
    "gpt2_op_attention_bwd_stored": ([ct.c_void_p, ct.c_void_p, ct.c_void_p, ct.c_void_p, ct.c_int, ct.c_int,
                                      ct.c_int, ct.c_int, ct.c_void_p, ct.c_void_p, ct.c_void_p], ct.c_int),
    "gpt2_attention_ds_bytes": ([ct.c_int, ct.c_int, ct.c_int], ct.c_size_t),
    "gpt2_op_embedding_fwd": ([ct.c_void_p, ct.c_void_p, ct.c_void_p, ct.c_int, ct.c_int, ct.c_int, ct.c_int,
                               ct.c_void_p, ct.c_void_p], ct.c_int),
    "gpt2_op_token_buckets": ([ct.c_void_p, ct.c_int, ct.c_int, ct.c_void_p, ct.c_void_p, ct.c_void_p,
                               ct.POINTER(ct.c_int32), ct.c_void_p], ct.c_int),
    "gpt2_op_embedding_bwd": ([ct.c_void_p, ct.c_void_p, ct.c_int, ct.c_int, ct.c_int, ct.c_int, ct.c_void_p,
                               ct.c_void_p, ct.c_void_p], ct.c_int),
    "gpt2_op_cross_entropy": ([ct.c_int, ct.c_void_p, ct.c_int64, ct.c_int, ct.c_int, ct.c_void_p, ct.c_float,
                               ct.c_void_p, ct.c_void_p], ct.c_int),
    "gpt2_op_attention_bwd_noalloc": ([ct.c_int, ct.c_void_p, ct.c_void_p, ct.c_void_p, ct.c_void_p, ct.c_int,
                                       ct.c_int, ct.c_int, ct.c_int, ct.c_void_p, ct.c_void_p], ct.c_int),
    "gpt2_prefill": ([ct.c_void_p, ct.c_void_p, ct.c_int, ct.c_int, ct.c_void_p, ct.c_int64], ct.c_int),
    "gpt2_decode_step": ([ct.c_void_p, ct.c_void_p, ct.c_int, ct.c_void_p, ct.c_int64], ct.c_int),
    "gpt2_sample_topk": ([ct.c_void_p, ct.c_void_p, ct.c_int64, ct.c_int, ct.c_int, ct.c_float, ct.c_float,
                          ct.c_void_p, ct.c_void_p], ct.c_int),
    "gpt2_kv_length": ([ct.c_void_p, ct.POINTER(ct.c_int)], ct.c_int),
    "gpt2_synchronize": ([ct.c_void_p], ct.c_int),
    "gpt2_op_gemv": ([ct.c_void_p, ct.c_int64, ct.c_int, ct.c_void_p, ct.c_int, ct.c_int, ct.c_int, ct.c_void_p,
                      ct.c_void_p, ct.c_int64, ct.c_void_p, ct.c_int64, ct.c_void_p, ct.c_void_p, ct.c_int, ct.c_int,
                      ct.POINTER(ct.c_float), ct.c_void_p], ct.c_int),
    "gpt2_op_sample_topk": ([ct.c_void_p, ct.c_int64, ct.c_int, ct.c_int, ct.c_int, ct.c_float, ct.c_float,
                             ct.c_void_p, ct.c_void_p, ct.c_void_p], ct.c_int),
    "gpt2_op_bounded_wait_check": ([ct.c_int, ct.c_ulonglong, ct.c_void_p], ct.c_int),
    "gpt2_grad_sumsq": ([ct.c_void_p, ct.c_int64, ct.c_int64, ct.c_void_p], ct.c_int),
    "gpt2_step_range": ([ct.c_void_p, ct.c_float, ct.c_float, ct.c_float, ct.c_float, ct.c_int64, ct.c_int64,
                         ct.c_void_p, ct.c_void_p], ct.c_int),
    "gpt2_param_buffer": ([ct.c_void_p, ct.POINTER(ct.c_void_p), ct.POINTER(ct.c_int64)], ct.c_int),
    "gpt2_refresh_shadow": ([ct.c_void_p], ct.c_int),
    "gpt2_storage_layout": ([ct.POINTER(_Config), ct.c_int, ct.c_char_p, ct.c_int, ct.POINTER(ct.c_int64),
                             ct.POINTER(ct.c_int64), ct.POINTER(ct.c_int), ct.POINTER(ct.c_int64)], ct.c_int),
    "gpt2_set_grad_events": ([ct.c_void_p, ct.POINTER(ct.c_void_p), ct.c_int], ct.c_int),
    "gpt2_read_loss": ([ct.c_void_p, ct.POINTER(ct.c_float)], ct.c_int),
    "gpt2_op_last_error": ([], ct.c_char_p),
}


def lib() -> ct.CDLL:
    """Load libgpt2_b200.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m train_step_b200.build` "
                               "(there is no CPU fallback)")
        L = ct.CDLL(LIB_PATH)
        for name, (args, res) in _SYMBOLS.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def exported_symbols() -> list[str]:
    return list(_SYMBOLS)


def _ptr(x):
    """Address of a torch tensor, numpy array or None."""
    if x is None:
        return None
    if isinstance(x, np.ndarray):
        return x.ctypes.data
    return x.data_ptr()


def _stream(stream=None):
    if stream is not None:
        return stream
    import torch
    return torch.cuda.current_stream().cuda_stream


def _op(code: int) -> None:
    if code != 0:
        raise Gpt2Error(code, lib().gpt2_op_last_error().decode())


@dataclass
class Config:
    L: int
    H: int
    C: int
    T: int
    V: int
    tied: int = 1
    qkv_bias: int = 1
    dtype: int = BF16
    B_max: int = 1

    def c(self) -> _Config:
        return _Config(self.L, self.H, self.C, self.T, self.V, self.tied, self.qkv_bias, self.dtype, self.B_max)


def storage_layout(cfg: Config):
    """Host-side storage layout of a configuration (no GPU needed): a list of
    (name, offset, length, bucket) per tensor in canonical order, and the storage length."""
    c = cfg.c()
    name = ct.create_string_buffer(64)
    off, n, ns = ct.c_int64(), ct.c_int64(), ct.c_int64()
    b = ct.c_int()
    out = []
    i = 0
    while lib().gpt2_storage_layout(ct.byref(c), i, name, 64, ct.byref(off), ct.byref(n), ct.byref(b),
                                    ct.byref(ns)) == 0:
        out.append((name.value.decode(), off.value, n.value, b.value))
        i += 1
    if not out:
        raise Gpt2Error(-1, "invalid configuration")
    return out, ns.value


def bucket_ranges(cfg: Config):
    """Storage ranges [(offset, length), ...] of each gradient bucket 0 .. L (adjacent
    tensors of one bucket merged, the padding between them included)."""
    layout, _ = storage_layout(cfg)
    per = [[] for _ in range(cfg.L + 1)]
    for _, off, n, b in sorted(layout, key=lambda t: t[1]):
        r = per[b]
        if r and r[-1][0] + r[-1][1] >= off - 63:  # contiguous up to the 64-float alignment
            r[-1] = (r[-1][0], off + n - r[-1][0])
        else:
            r.append((off, n))
    return per


class GPT2:
    """One model handle: parameters, gradients, Adam state and activations on the GPU."""

    def __init__(self, cfg: Config, seed: int = 42, stream=None):
        self.cfg = cfg
        h = ct.c_void_p()
        c = cfg.c()
        rc = lib().gpt2_create(ct.byref(c), seed, ct.byref(h))
        if rc != 0:
            raise Gpt2Error(rc, "gpt2_create failed")
        self.h = h
        if stream is not None:
            self._check(lib().gpt2_set_stream(self.h, stream))

    def _check(self, rc: int) -> None:
        if rc != 0:
            raise Gpt2Error(rc, lib().gpt2_last_error(self.h).decode())

    def close(self) -> None:
        if getattr(self, "h", None):
            lib().gpt2_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def set_stream(self, stream) -> None:
        self._check(lib().gpt2_set_stream(self.h, stream))

    def forward_backward(self, tokens, targets, want_loss: bool = True):
        B, T = tokens.shape
        loss = ct.c_float()
        self._check(lib().gpt2_forward_backward(self.h, _ptr(tokens), _ptr(targets), B, T,
                                                ct.byref(loss) if want_loss else None))
        return loss.value if want_loss else None

    def read_loss(self) -> float:
        """Mean loss of the most recent forward_backward / forward (waits for the GPU)."""
        loss = ct.c_float()
        self._check(lib().gpt2_read_loss(self.h, ct.byref(loss)))
        return loss.value

    def forward(self, tokens, targets):
        B, T = tokens.shape
        loss = ct.c_float()
        self._check(lib().gpt2_forward(self.h, _ptr(tokens), _ptr(targets), B, T, ct.byref(loss)))
        return loss.value

    def step(self, lr: float, wd: float, beta1: float = 0.9, beta2: float = 0.95, want_norm: bool = True):
        n = ct.c_float()
        self._check(lib().gpt2_step(self.h, lr, wd, beta1, beta2, ct.byref(n) if want_norm else None))
        return n.value if want_norm else None

    def zero_grad(self) -> None:
        self._check(lib().gpt2_zero_grad(self.h))

    @property
    def num_params(self) -> int:
        n = ct.c_int64()
        self._check(lib().gpt2_num_params(self.h, ct.byref(n)))
        return n.value

    def tensors(self):
        out = []
        name = ct.create_string_buffer(64)
        r, c, o = ct.c_int64(), ct.c_int64(), ct.c_int64()
        nd = ct.c_int()
        i = 0
        while lib().gpt2_tensor_info(self.h, i, name, 64, ct.byref(r), ct.byref(c), ct.byref(nd), ct.byref(o)) == 0:
            shape = (r.value, c.value) if nd.value == 2 else (r.value,)
            out.append((name.value.decode(), shape, o.value))
            i += 1
        return out

    def get_params(self) -> np.ndarray:
        out = np.empty(self.num_params, np.float32)
        self._check(lib().gpt2_get_params(self.h, out.ctypes.data, out.size))
        return out

    def set_params(self, p) -> None:
        p = np.ascontiguousarray(p, np.float32)
        self._check(lib().gpt2_set_params(self.h, p.ctypes.data, p.size))

    def get_grads(self) -> np.ndarray:
        out = np.empty(self.num_params, np.float32)
        self._check(lib().gpt2_get_grads(self.h, out.ctypes.data, out.size))
        return out

    def get_adam(self):
        m = np.empty(self.num_params, np.float32)
        v = np.empty(self.num_params, np.float32)
        t = ct.c_int64()
        self._check(lib().gpt2_get_adam(self.h, m.ctypes.data, v.ctypes.data, m.size, ct.byref(t)))
        return m, v, t.value

    def set_adam(self, m: np.ndarray, v: np.ndarray, t: int) -> None:
        """Restore the Adam moments (canonical order) and step count."""
        m = np.ascontiguousarray(m, dtype=np.float32)
        v = np.ascontiguousarray(v, dtype=np.float32)
        if m.size != self.num_params or v.size != self.num_params:
            raise ValueError("Adam moments must have num_params entries")
        self._check(lib().gpt2_set_adam(self.h, m.ctypes.data, v.ctypes.data, m.size, int(t)))

    def grad_buffer(self):
        """(device address, length in floats) of the flat gradient storage."""
        p = ct.c_void_p()
        n = ct.c_int64()
        self._check(lib().gpt2_grad_buffer(self.h, ct.byref(p), ct.byref(n)))
        return p.value, n.value

    @staticmethod
    def _device_view(ptr: int, n: int):
        import torch

        class _View:
            pass

        v = _View()
        v.__cuda_array_interface__ = {"shape": (n,), "typestr": "<f4", "data": (ptr, False), "version": 3}
        return torch.as_tensor(v, device="cuda")

    def set_grad_events(self, events) -> None:
        """Arm the next forward_backward to record events[b] (torch.cuda.Event objects that
        have been recorded once, or raw handles) as gradient bucket b completes; [] cancels."""
        hs = [e.cuda_event if hasattr(e, "cuda_event") else int(e) for e in events]
        arr = (ct.c_void_p * max(1, len(hs)))(*hs)
        self._check(lib().gpt2_set_grad_events(self.h, arr, len(hs)))

    def grad_tensor(self):
        """Zero-copy fp32 CUDA tensor over the flat gradient storage (the library's padded
        layout), e.g. for a data-parallel all-reduce between micro-batch accumulation and
        the optimizer step."""
        return self._device_view(*self.grad_buffer())

    def param_buffer(self):
        """(device address, length in floats) of the flat fp32 parameter storage."""
        p = ct.c_void_p()
        n = ct.c_int64()
        self._check(lib().gpt2_param_buffer(self.h, ct.byref(p), ct.byref(n)))
        return p.value, n.value

    def param_tensor(self):
        """Zero-copy fp32 CUDA tensor over the flat parameter storage (padded layout)."""
        return self._device_view(*self.param_buffer())

    def grad_sumsq(self, lo: int, hi: int, out) -> None:
        """out (a CUDA float64 tensor of one element) = sum of squares of the accumulated
        gradient sum over storage [lo, hi); asynchronous."""
        self._check(lib().gpt2_grad_sumsq(self.h, int(lo), int(hi), _ptr(out)))

    def step_range(self, lr: float, wd: float, beta1: float, beta2: float, lo: int, hi: int, sumsq,
                   want_norm: bool = False):
        """The optimizer step on storage [lo, hi) with the whole gradient's squared norm in
        sumsq (a CUDA float64 tensor of one element); returns the pre-clip norm if asked."""
        n = ct.c_float()
        self._check(lib().gpt2_step_range(self.h, lr, wd, beta1, beta2, int(lo), int(hi), _ptr(sumsq),
                                          ct.byref(n) if want_norm else None))
        return n.value if want_norm else None

    def refresh_shadow(self) -> None:
        self._check(lib().gpt2_refresh_shadow(self.h))

    def profile(self, enable: bool) -> None:
        self._check(lib().gpt2_profile(self.h, int(enable)))

    def profile_read(self) -> dict:
        """{category: (ms, launches, flops, bytes)} of the recorded launches."""
        out = {}
        name = ct.create_string_buffer(64)
        ms, fl, by = ct.c_double(), ct.c_double(), ct.c_double()
        n = ct.c_int64()
        i = 0
        while lib().gpt2_profile_read(self.h, i, name, 64, ct.byref(ms), ct.byref(n), ct.byref(fl), ct.byref(by)) == 0:
            out[name.value.decode()] = (ms.value, n.value, fl.value, by.value)
            i += 1
        return out

    def launch_count(self) -> int:
        n = ct.c_int64()
        self._check(lib().gpt2_launch_count(self.h, ct.byref(n)))
        return n.value

    # ---- generation (bf16 models) ----
    # The library runs on the handle's stream (its own unless one was given). With
    # sync=True (the default) a call first waits for torch's current stream (so inputs made
    # there are ready) and returns after its own kernels have finished, so its outputs can
    # be used from any stream; sync=False does neither: inputs must come from the handle's
    # stream and outputs stay in flight there (call synchronize() before using them
    # elsewhere).
    def synchronize(self) -> None:
        self._check(lib().gpt2_synchronize(self.h))

    def _logits_buffer(self, B: int, out=None):
        import torch
        if out is None:
            out = torch.empty(B, self.cfg.V, device="cuda", dtype=torch.float32)
        return out

    def prefill(self, tokens, logits_out=None):
        """Forward of B prompts (int32 [B, T0], host or CUDA), fill the key/value cache,
        return the fp32 logits [B, V] of each prompt's last position (a CUDA tensor).
        Always synchronises (before and after, as sync=True does)."""
        import torch
        B, T0 = tokens.shape
        out = self._logits_buffer(B, logits_out)
        torch.cuda.current_stream().synchronize()
        self._check(lib().gpt2_prefill(self.h, _ptr(tokens), B, T0, _ptr(out), out.stride(0)))
        return out

    def decode_step(self, tokens, logits_out=None, sync: bool = True):
        """Append one token per sequence (int32 [B]) at the next cache position; return
        the fp32 logits [B, V] of that position."""
        import torch
        B = tokens.shape[0]
        out = self._logits_buffer(B, logits_out)
        if sync:
            torch.cuda.current_stream().synchronize()
        self._check(lib().gpt2_decode_step(self.h, _ptr(tokens), B, _ptr(out), out.stride(0)))
        if sync:
            self.synchronize()
        return out

    def sample_topk(self, logits, k: int, temperature: float, top_p: float, u, out=None, sync: bool = True):
        """One index per logits row (int32 CUDA tensor); u: float64 CUDA tensor [rows] in [0, 1)."""
        import torch
        rows = logits.shape[0]
        if out is None:
            out = torch.empty(rows, device="cuda", dtype=torch.int32)
        if sync:
            torch.cuda.current_stream().synchronize()
        self._check(lib().gpt2_sample_topk(self.h, _ptr(logits), logits.stride(0), rows, k, temperature, top_p,
                                           _ptr(u), _ptr(out)))
        if sync:
            self.synchronize()
        return out

    @property
    def kv_length(self) -> int:
        n = ct.c_int()
        self._check(lib().gpt2_kv_length(self.h, ct.byref(n)))
        return n.value

    def generate(self, prompt, max_new_tokens: int, k: int = 50, temperature: float = 1.0, top_p: float = 1.0,
                 seed: int = 0):
        """Sample max_new_tokens tokens after each prompt row (int32 [B, T0]); returns the
        int32 CUDA tensor [B, T0 + max_new_tokens]. The uniform draws u come from numpy's
        PCG64 seeded with `seed`, shape [max_new_tokens, B], and are passed to the sampler;
        the loop stays on the handle's stream and synchronises once at the end."""
        import torch
        B, T0 = prompt.shape
        if T0 + max_new_tokens > self.cfg.T + 1:
            raise ValueError("prompt plus new tokens exceed the block size + 1")
        prompt = torch.as_tensor(prompt, dtype=torch.int32).cuda().contiguous()
        if max_new_tokens == 0:
            return prompt
        u = torch.from_numpy(np.random.default_rng(seed).random((max_new_tokens, B))).cuda()
        new = torch.empty(max_new_tokens, B, device="cuda", dtype=torch.int32)
        torch.cuda.current_stream().synchronize()  # inputs made on torch's stream are ready
        logits = self.prefill(prompt)
        for s in range(max_new_tokens):
            self.sample_topk(logits, k, temperature, top_p, u[s], out=new[s], sync=False)
            if s + 1 < max_new_tokens:
                self.decode_step(new[s], logits_out=logits, sync=False)
        self.synchronize()
        return torch.cat([prompt, new.t()], dim=1)


# ---------------------------------------------------------------------------
# op-level wrappers (torch CUDA tensors in, results written in place)
# ---------------------------------------------------------------------------
def _dt(t) -> int:
    import torch
    return BF16 if t.dtype == torch.bfloat16 else FP32


def gemm(A, B, out, *, M, N, K, lda, ldb, ldo, a_mn=False, b_mn=False, epilogue=EPI_F32, out2=None, ldo2=0,
         bias=None, aux=None, ld_aux=0, accumulate=False, ksplit=1, stream=None):
    _op(lib().gpt2_op_gemm(_dt(A), _ptr(A), lda, int(a_mn), _ptr(B), ldb, int(b_mn), M, N, K, epilogue, _ptr(out),
                           ldo, _ptr(out2), ldo2, _ptr(bias), _ptr(aux), ld_aux, int(accumulate), ksplit,
                           _stream(stream)))


def gemm_bench(A, B, out, *, M, N, K, lda, ldb, ldo, a_mn=False, b_mn=False, epilogue=EPI_F32, out2=None, ldo2=0,
               bias=None, aux=None, ld_aux=0, accumulate=False, ksplit=1, bn=0, pair=-1, iters=20,
               stream=None) -> float:
    """Average milliseconds of the bf16 tensor-core GEMM over `iters` back-to-back launches
    (pair: -1 library choice, 0 one CTA per tile, 1 two-CTA 256 x 256 tiles)."""
    ms = ct.c_float()
    _op(lib().gpt2_op_gemm_bench(_ptr(A), lda, int(a_mn), _ptr(B), ldb, int(b_mn), M, N, K, epilogue, _ptr(out), ldo,
                                 _ptr(out2), ldo2, _ptr(bias), _ptr(aux), ld_aux, int(accumulate), ksplit, bn, pair,
                                 iters, ct.byref(ms), _stream(stream)))
    return ms.value


def layernorm_fwd(x, g, b, y, mean, rstd, stream=None):
    N, C = x.shape
    _op(lib().gpt2_op_layernorm_fwd(_dt(y), _ptr(x), _ptr(g), _ptr(b), N, C, _ptr(y), _ptr(mean), _ptr(rstd),
                                    _stream(stream)))


def layernorm_bwd(dy, x, g, mean, rstd, dres, dres_act, dg, db, accumulate=False, accumulate_params=False,
                  dtype=None, stream=None):
    N, C = x.shape
    dt = dtype if dtype is not None else (_dt(dres_act) if dres_act is not None else FP32)
    _op(lib().gpt2_op_layernorm_bwd(dt, _ptr(dy), _ptr(x), _ptr(g), _ptr(mean), _ptr(rstd), N, C, _ptr(dres),
                                    _ptr(dres_act), int(accumulate), _ptr(dg), _ptr(db), int(accumulate_params),
                                    _stream(stream)))


def gemv(x, W, out, *, B, N, K, epilogue, ldx=None, ldo=None, bias=None, resid=None, ldr=0, ln_g=None, ln_b=None,
         iters=1, pdl=False, stream=None):
    """Skinny product of a generation step (see gpt2_op_gemv); returns ms per launch when
    iters > 1."""
    ms = ct.c_float()
    _op(lib().gpt2_op_gemv(_ptr(x), x.stride(0) if ldx is None else ldx, B, _ptr(W), N, K, epilogue, _ptr(bias),
                           _ptr(out), out.stride(0) if ldo is None else ldo, _ptr(resid), ldr, _ptr(ln_g),
                           _ptr(ln_b), iters, int(pdl), ct.byref(ms), _stream(stream)))
    return ms.value if iters > 1 else None


def sample_topk(logits, V, k, temperature, top_p, u, out, stream=None):
    """Op-level sampler: logits fp32 [rows, ld] (ld = stride), u float64 [rows], out int32 [rows]."""
    _op(lib().gpt2_op_sample_topk(_ptr(logits), logits.stride(0), logits.shape[0], V, k, temperature, top_p,
                                  _ptr(u), _ptr(out), _stream(stream)))


def attention_fwd(qkv, out, lse, B, T, NH, hd, stream=None):
    _op(lib().gpt2_op_attention_fwd(_dt(qkv), _ptr(qkv), B, T, NH, hd, _ptr(out), _ptr(lse), _stream(stream)))


def attention_bwd(qkv, out, dout, lse, dqkv, B, T, NH, hd, stream=None):
    _op(lib().gpt2_op_attention_bwd(_dt(qkv), _ptr(qkv), _ptr(out), _ptr(dout), _ptr(lse), B, T, NH, hd,
                                    _ptr(dqkv), _stream(stream)))


def attention_ds_bytes(B, T, NH):
    return lib().gpt2_attention_ds_bytes(B, T, NH)


def attention_bwd_stored(qkv, out, dout, lse, dqkv, ds, B, T, NH, hd, stream=None):
    """The training step's attention backward (bf16): dS^T tiles kept in ds
    (attention_ds_bytes(B, T, NH) bytes of device memory) and dQ computed from them."""
    _op(lib().gpt2_op_attention_bwd_stored(_ptr(qkv), _ptr(out), _ptr(dout), _ptr(lse), B, T, NH, hd, _ptr(dqkv),
                                           _ptr(ds), _stream(stream)))


def attention_bwd_noalloc(qkv, out, dout, lse, dqkv, B, T, NH, hd, stream=None):
    """Attention backward with its scratch in a fixed device array: for callers
    that may not allocate device memory themselves (see include/gpt2.h)."""
    _op(lib().gpt2_op_attention_bwd_noalloc(_dt(qkv), _ptr(qkv), _ptr(out), _ptr(dout), _ptr(lse), B, T, NH, hd,
                                            _ptr(dqkv), _stream(stream)))


def embedding_fwd(tokens, wte, wpe, x0, stream=None):
    B, T = tokens.shape
    V, C = wte.shape
    _op(lib().gpt2_op_embedding_fwd(_ptr(tokens), _ptr(wte), _ptr(wpe), B, T, C, V, _ptr(x0), _stream(stream)))


def token_buckets(tokens, V, sorted_pos, seg_id, seg_start, stream=None) -> int:
    n = ct.c_int32()
    _op(lib().gpt2_op_token_buckets(_ptr(tokens), tokens.numel(), V, _ptr(sorted_pos), _ptr(seg_id), _ptr(seg_start),
                                    ct.byref(n), _stream(stream)))
    return n.value


def embedding_bwd(tokens, dx0, dwte, dwpe, stream=None):
    B, T = tokens.shape
    V, C = dwte.shape
    _op(lib().gpt2_op_embedding_bwd(_ptr(tokens), _ptr(dx0), B, T, C, V, _ptr(dwte), _ptr(dwpe), _stream(stream)))


def cross_entropy(logits, V, targets, scale, row_loss, stream=None):
    N, ld = logits.shape
    _op(lib().gpt2_op_cross_entropy(_dt(logits), _ptr(logits), ld, N, V, _ptr(targets), scale, _ptr(row_loss),
                                    _stream(stream)))


def bounded_wait_check(arrive: bool, limit_ns: int, stream=None) -> None:
    """The library's bounded device-side wait on a barrier that is completed (arrive) or
    never completed; raises Gpt2Error(GPT2_ERR_TIMEOUT) when the wait gives up."""
    _op(lib().gpt2_op_bounded_wait_check(int(arrive), int(limit_ns), _stream(stream)))

