"""Pins of the oracle's projection (x W of Algorithm 1, lines 1-2): one-hot
rows of x pick rows of W, a brute-force sum over d_model on a tiny case,
and bf16 widening that is exact (values a bf16 holds come back unchanged)."""
from __future__ import annotations

import numpy as np

import oracle
from block_sparse_gqa_idx_b200 import inputs


def test_one_hot_rows_pick_rows_of_w():
    rng = np.random.default_rng(0)
    d, n = 16, 24
    w = inputs.bf16_bits(rng.standard_normal((d, n)).astype(np.float32))
    x = np.zeros((d, d), np.float32)
    x[np.arange(d), np.arange(d)[::-1]] = 1.0
    y = oracle.project(inputs.bf16_bits(x), w)
    assert np.array_equal(y, inputs.bf16_to_f32(w)[::-1].astype(np.float64))


def test_brute_force_sum_on_a_tiny_case():
    rng = np.random.default_rng(1)
    T, d, n = 3, 5, 4
    xb = inputs.bf16_bits(rng.standard_normal((T, d)).astype(np.float32))
    wb = inputs.bf16_bits(rng.standard_normal((d, n)).astype(np.float32))
    xf, wf = inputs.bf16_to_f32(xb), inputs.bf16_to_f32(wb)
    y = oracle.project(xb, wb)
    for t in range(T):
        for j in range(n):
            s = 0.0
            for c in range(d):
                s += float(xf[t, c]) * float(wf[c, j])
            assert abs(y[t, j] - s) <= 1e-12 * max(1.0, abs(s))


def test_powers_of_two_are_exact():
    x = inputs.bf16_bits(np.array([[0.5, 2.0, -4.0]], np.float32))
    w = inputs.bf16_bits(np.array([[1.0], [0.25], [0.125]], np.float32))
    assert oracle.project(x, w).tolist() == [[0.5 + 0.5 - 0.5]]
