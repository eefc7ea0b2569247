"""Pins of the oracle's temperature / top-k / top-p sampler (CPU only).

The sampler is checked against hand-worked draws (tests/golden), closed forms (uniform
logits, k = 1), an independent formulation of the draw probabilities (a stable argsort
plus a float64 softmax of the kept logits, integrated over a grid of u), and its
tie and signed-zero rules.
"""
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "sampling_worked_example.txt")


def _golden():
    logits, cases = None, []
    for line in open(GOLDEN):
        line = line.split("#", 1)[0].strip()
        if not line:
            continue
        if line.startswith("logits"):
            logits = [float(x) for x in line.split("=", 1)[1].split()]
            continue
        k, t, p, u, idx = line.split()
        cases.append((int(k), float(t), float(p), float(u), int(idx)))
    return logits, cases


def test_hand_worked_draws():
    z, cases = _golden()
    assert len(cases) >= 9
    for k, t, p, u, idx in cases:
        assert oracle.sample_topk(z, k, t, p, u) == idx, (k, t, p, u)


def test_uniform_logits_closed_form():
    # equal logits: the first k indices carry weight 1 each, so the draw is index floor(u k)
    z = np.zeros(10, np.float32)
    for k in (1, 3, 4, 10):
        for u in (0.0, 0.13, 0.49, 0.74, 0.999):
            assert oracle.sample_topk(z, k, 0.8, 1.0, u) == math.floor(u * k)


def test_k1_is_first_argmax():
    rng = np.random.default_rng(1)
    z = rng.integers(0, 5, 40).astype(np.float32)
    first = int(np.flatnonzero(z == z.max())[0])
    for u in (0.0, 0.5, 0.999):
        assert oracle.sample_topk(z, 1, 2.0, 1.0, u) == first


def test_signed_zero_ties_by_index():
    assert oracle.sample_topk([-0.0, 0.0], 1, 1.0, 1.0, 0.5) == 0
    assert oracle.sample_topk([0.0, -0.0], 1, 1.0, 1.0, 0.5) == 0


@pytest.mark.parametrize("k,temp,top_p", [(7, 1.0, 1.0), (7, 0.6, 1.0), (12, 1.7, 0.85), (30, 1.0, 0.5)])
def test_draw_frequencies_match_softmax(k, temp, top_p):
    # probabilities by another route: numpy's stable argsort of -z for the kept set and a
    # float64 softmax, nucleus cut on the normalised cumulative probabilities
    rng = np.random.default_rng(k)
    z = (rng.standard_normal(30) * 2).astype(np.float32)
    keep = np.argsort(-z.astype(np.float64), kind="stable")[:k]
    e = np.exp(z[keep].astype(np.float64) / temp - np.max(z[keep].astype(np.float64) / temp))
    p = e / e.sum()
    if top_p < 1.0:
        m = int(np.searchsorted(np.cumsum(p), np.float32(top_p) - 1e-12)) + 1
        keep, p = keep[:m], p[:m] / p[:m].sum()
    n = 20000
    counts = {}
    for i in range(n):
        j = oracle.sample_topk(z, k, temp, top_p, (i + 0.5) / n)
        counts[j] = counts.get(j, 0) + 1
    assert set(counts) <= set(keep.tolist())
    for idx, prob in zip(keep.tolist(), p):
        assert abs(counts.get(idx, 0) / n - prob) <= 1.5 / n, (idx, prob)


def test_draw_is_monotone_in_u():
    rng = np.random.default_rng(5)
    z = (rng.standard_normal(50)).astype(np.float32)
    ranked = sorted(range(50), key=lambda i: (-z[i], i))
    pos = [ranked.index(oracle.sample_topk(z, 20, 1.3, 1.0, u)) for u in np.linspace(0, 0.9999, 200)]
    assert pos == sorted(pos)
