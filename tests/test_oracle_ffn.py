"""Pins of the oracle's blockwise feed-forward network (oracle/feedforward.py).

Pinned to things other than its own formula: silu's closed-form values and
limits, torch's float64 silu (a library routine), a pure-Python loop
restatement on tiny inputs, zero and linearity properties of the gated
network, and chunk invariance.
"""

from __future__ import annotations

import math

import numpy as np
import torch

import oracle


def test_silu_closed_forms_and_library():
    assert oracle.silu(np.array([0.0]))[0] == 0.0
    assert abs(oracle.silu(np.array([1.0]))[0] - 1.0 / (1.0 + math.exp(-1.0))) < 1e-16
    assert abs(oracle.silu(np.array([-2.0]))[0] - (-2.0 / (1.0 + math.exp(2.0)))) < 1e-16
    big = oracle.silu(np.array([800.0, -800.0]))
    assert big[0] == 800.0 and big[1] == 0.0 and np.all(np.isfinite(big))
    a = np.random.default_rng(1).standard_normal(1000) * 8
    ref = torch.nn.functional.silu(torch.from_numpy(a)).numpy()
    np.testing.assert_allclose(oracle.silu(a), ref, rtol=1e-14, atol=1e-300)


def _loops(x, w1, w3, w2):
    T, dm = x.shape
    dff = w1.shape[0]
    y = [[0.0] * w2.shape[0] for _ in range(T)]
    for t in range(T):
        h = []
        for f in range(dff):
            a = sum(x[t][i] * w1[f][i] for i in range(dm))
            g = sum(x[t][i] * w3[f][i] for i in range(dm))
            h.append(a / (1.0 + math.exp(-a)) * g)
        for o in range(w2.shape[0]):
            y[t][o] = sum(h[f] * w2[o][f] for f in range(dff))
    return np.array(y)


def _weights(seed, T=9, dm=6, dff=10):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((T, dm)), rng.standard_normal((dff, dm)) / 2, rng.standard_normal((dff, dm)) / 2,
            rng.standard_normal((dm, dff)) / 3)


def test_ffn_matches_loops_on_tiny_inputs():
    x, w1, w3, w2 = _weights(2)
    np.testing.assert_allclose(oracle.blockwise_feedforward(x, w1, w3, w2, chunk_size=4), _loops(x, w1, w3, w2),
                               rtol=1e-12, atol=1e-12)


def test_ffn_chunk_invariance_and_hidden():
    x, w1, w3, w2 = _weights(3, T=37)
    full = oracle.blockwise_feedforward(x, w1, w3, w2)
    for c in (1, 5, 16, 37, 100):
        np.testing.assert_allclose(oracle.blockwise_feedforward(x, w1, w3, w2, chunk_size=c), full, rtol=1e-13,
                                   atol=1e-13)
    y, h = oracle.blockwise_feedforward(x, w1, w3, w2, chunk_size=8, return_hidden=True)
    np.testing.assert_allclose(h @ w2.T, y, rtol=1e-13, atol=1e-13)


def test_ffn_zero_and_linearity():
    x, w1, w3, w2 = _weights(4)
    assert np.all(oracle.blockwise_feedforward(np.zeros_like(x), w1, w3, w2) == 0)
    assert np.all(oracle.blockwise_feedforward(x, w1, np.zeros_like(w3), w2) == 0)
    y = oracle.blockwise_feedforward(x, w1, w3, w2)
    np.testing.assert_allclose(oracle.blockwise_feedforward(x, w1, 3 * w3, w2), 3 * y, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(oracle.blockwise_feedforward(x, w1, w3, -2 * w2), -2 * y, rtol=1e-12, atol=1e-12)
    # the gate is silu(x W1^T), not linear in W1: doubling W1 does not double y
    assert not np.allclose(oracle.blockwise_feedforward(x, 2 * w1, w3, w2), 2 * y)
