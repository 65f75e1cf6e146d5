"""Pins of the oracle's output projection (y = x W^T + b): closed forms that a
transposed operand, a dropped bias or a wrong axis would break."""
import numpy as np

import oracle


def test_identity_weight_returns_input():
    x = np.random.default_rng(0).standard_normal((7, 16))
    assert np.array_equal(oracle.project(x, np.eye(16)), x)


def test_zero_weight_returns_bias():
    b = np.arange(32, dtype=np.float64)
    y = oracle.project(np.ones((5, 8)), np.zeros((32, 8)), b)
    assert np.array_equal(y, np.broadcast_to(b, (5, 32)))


def test_permutation_selects_input_columns():
    """Row n of the weight with a single 1 at column p(n) copies input column
    p(n) to output column n: the weight is indexed [out, in]."""
    rng = np.random.default_rng(1)
    x = rng.standard_normal((9, 12))
    perm = rng.permutation(12)[:8]
    w = np.zeros((8, 12))
    w[np.arange(8), perm] = 1.0
    assert np.array_equal(oracle.project(x, w), x[:, perm])


def test_composition():
    """Two projections in a row equal one with the product weight."""
    rng = np.random.default_rng(2)
    x = rng.standard_normal((6, 10))
    w1, w2 = rng.standard_normal((8, 10)), rng.standard_normal((4, 8))
    np.testing.assert_allclose(oracle.project(oracle.project(x, w1), w2),
                               oracle.project(x, w2 @ w1), rtol=1e-12, atol=1e-12)
