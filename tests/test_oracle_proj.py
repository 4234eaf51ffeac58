"""Pins of the oracle's projections (q = W_Q x, k = W_K x, v = W_V x, gates = sigmoid(W x);
paper-read, section 2, second pillar, GLA paragraph) against things other than its own code:
exact brute force on grid values, the identity weight, and the sigmoid's fixed points."""
from fractions import Fraction

import numpy as np

import oracle

RNG = np.random.default_rng(4242)


def grid(shape, scale=8):
    return (RNG.integers(-16, 17, size=shape) / scale).astype(np.float32)


def test_projection_equals_exact_brute_force():
    M, K, N = 3, 5, 4
    x, w = grid((M, K)), grid((N, K))
    y = oracle.proj(x, w)
    for r in range(M):
        for n in range(N):
            exact = sum(Fraction(float(x[r, c])) * Fraction(float(w[n, c])) for c in range(K))
            assert y[r, n] == float(exact)


def test_identity_weight_returns_the_input():
    x = RNG.standard_normal((7, 16)).astype(np.float32)
    y = oracle.proj(x, np.eye(16, dtype=np.float32))
    assert np.array_equal(y, x.astype(np.float64))


def test_sigmoid_columns_fixed_points_and_symmetry():
    x = RNG.standard_normal((6, 8)).astype(np.float32)
    w = RNG.standard_normal((5, 8)).astype(np.float32)
    w[2] = 0.0             # zero row -> sigmoid(0) = 1/2 exactly
    w[4] = -w[3]           # negated row -> sigmoid(-y) = 1 - sigmoid(y)
    y = oracle.proj(x, w, sigmoid_cols=(2, 5))
    assert np.all(y[:, 2] == 0.5)
    np.testing.assert_allclose(y[:, 4], 1.0 - y[:, 3], rtol=0, atol=1e-15)
    raw = oracle.proj(x, w)
    np.testing.assert_array_equal(y[:, :2], raw[:, :2])
    assert np.all((y[:, 3] > 0) & (y[:, 3] < 1))
    assert np.all((y[:, 3] > 0.5) == (raw[:, 3] > 0))


def test_stacked_weights_and_row_selection():
    x = grid((9, 12))
    wq, wk = grid((4, 12)), grid((6, 12))
    y = oracle.proj(x, np.concatenate([wq, wk]))
    np.testing.assert_array_equal(y[:, :4], oracle.proj(x, wq))
    np.testing.assert_array_equal(y[:, 4:], oracle.proj(x, wk))
    rows = [8, 0, 3]
    np.testing.assert_array_equal(oracle.proj(x, wq, rows=rows), oracle.proj(x, wq)[rows])


def test_bias_shifts_logits_before_the_sigmoid():
    x = grid((4, 8))
    w = grid((3, 8))
    w[1] = 0.0
    b = np.array([0.5, 3.0, -1.25], dtype=np.float32)
    y = oracle.proj(x, w, sigmoid_cols=(1, 3), bias=b)
    raw = oracle.proj(x, w)
    np.testing.assert_array_equal(y[:, 0], raw[:, 0] + 0.5)
    np.testing.assert_allclose(y[:, 1], 1.0 / (1.0 + np.exp(-3.0)), rtol=0, atol=1e-16)
    np.testing.assert_allclose(y[:, 2], 1.0 / (1.0 + np.exp(-(raw[:, 2] - 1.25))), rtol=1e-15)
