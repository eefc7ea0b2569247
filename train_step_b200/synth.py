"""Seeded synthetic inputs for the GPT-2 training step.

This module only draws token ids. It holds none of the model's arithmetic, so
both the CUDA path (bench, smoke) and the float64 oracle's tests can use it.

The pages train on text corpora (Tiny Shakespeare for the character-level
model, OpenWebText / FineWeb-Edu / WikiText-103 for the BPE models). None is
available here, so these draws stand in for them:

* character-level data -> ids uniform over [0, V) (V = 65 for the tiny model);
* GPT-2 BPE text -> ids from a Zipf law, P(id = k) proportional to (k+1)^-s with
  s = 1.1 over [0, 50257), drawn by inverse-CDF lookup in a float64 cumulative
  table.

Randomness comes from splitmix64 (S. Vigna's published generator: the state
advances by the golden-ratio increment 0x9E3779B97F4A7C15 and each output is the
state passed through the published 64-bit finaliser). The i-th draw (i >= 0) of
the stream with seed s is finalise(s + (i + 1) * 0x9E3779B97F4A7C15) mod 2^64.
A uniform double in [0, 1) is the top 53 bits of a draw times 2^-53.

A micro-batch of B sequences of length T draws B*(T+1) ids from the stream with
seed ``base_seed + micro_batch_index``; tokens are buf[:, :T] and targets
buf[:, 1:] (next-token prediction).
"""
from __future__ import annotations

import functools

import numpy as np

GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def splitmix64_stream(seed: int, n: int) -> np.ndarray:
    """First ``n`` outputs of the splitmix64 stream started at ``seed`` (uint64)."""
    with np.errstate(over="ignore"):
        i = np.arange(1, n + 1, dtype=np.uint64)
        z = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + i * GOLDEN
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        z = z ^ (z >> np.uint64(31))
    return z


def uniform01(seed: int, n: int) -> np.ndarray:
    """``n`` float64 uniforms in [0, 1) from the top 53 bits of each draw."""
    return (splitmix64_stream(seed, n) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


@functools.lru_cache(maxsize=8)
def _zipf_cdf(vocab: int, s: float) -> np.ndarray:
    w = np.arange(1, vocab + 1, dtype=np.float64) ** (-s)
    c = np.cumsum(w)
    return c / c[-1]


def zipf_ids(seed: int, n: int, vocab: int = 50257, s: float = 1.1) -> np.ndarray:
    """``n`` ids in [0, vocab) with P(k) proportional to (k+1)^-s (int32)."""
    u = uniform01(seed, n)
    idx = np.searchsorted(_zipf_cdf(vocab, s), u, side="right")
    return np.minimum(idx, vocab - 1).astype(np.int32)


def uniform_ids(seed: int, n: int, vocab: int) -> np.ndarray:
    """``n`` ids uniform over [0, vocab) (int32)."""
    u = uniform01(seed, n)
    return np.minimum((u * vocab).astype(np.int64), vocab - 1).astype(np.int32)


def micro_batch(B: int, T: int, vocab: int, index: int = 0, base_seed: int = 1234,
                dist: str = "zipf") -> tuple[np.ndarray, np.ndarray]:
    """(tokens, targets), each int32 [B, T], for micro-batch ``index``.

    ``dist`` is "zipf" (BPE stand-in, s = 1.1) or "uniform" (char-level stand-in).
    """
    seed = base_seed + index
    n = B * (T + 1)
    if dist == "zipf":
        buf = zipf_ids(seed, n, vocab)
    elif dist == "uniform":
        buf = uniform_ids(seed, n, vocab)
    else:
        raise ValueError(f"unknown token distribution {dist!r}")
    buf = buf.reshape(B, T + 1)
    return np.ascontiguousarray(buf[:, :T]), np.ascontiguousarray(buf[:, 1:])
