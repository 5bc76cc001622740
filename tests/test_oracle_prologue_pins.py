"""Pins for the oracle's input prologue (CPU only): unit-norm keys and queries that
keep their direction, and the decay alpha = exp(-softplus(x)) against its closed
form 1 / (1 + e^x) and exact values of softplus."""
import math

import numpy as np

import oracle


def test_rows_become_unit_vectors_in_the_same_direction():
    rng = np.random.default_rng(21)
    q = rng.normal(size=(2, 5, 3, 8)) * 3.0
    k = rng.normal(size=(2, 5, 3, 8)) * 0.2
    qn, kn, _ = oracle.prologue(q, k, np.zeros_like(q))
    np.testing.assert_allclose(np.linalg.norm(qn, axis=-1), 1.0, rtol=0, atol=1e-14)
    np.testing.assert_allclose(np.linalg.norm(kn, axis=-1), 1.0, rtol=0, atol=1e-14)
    # same direction: <q_n, q> = |q|
    np.testing.assert_allclose((qn * q).sum(-1), np.linalg.norm(q, axis=-1), rtol=1e-13)
    np.testing.assert_allclose((kn * k).sum(-1), np.linalg.norm(k, axis=-1), rtol=1e-13)


def test_zero_row_stays_zero():
    q = np.zeros((1, 2, 1, 4))
    q[0, 1, 0] = [3.0, 0.0, 4.0, 0.0]
    qn, _, _ = oracle.prologue(q, q, np.zeros_like(q))
    assert np.all(qn[0, 0] == 0.0)
    np.testing.assert_allclose(qn[0, 1, 0], [0.6, 0.0, 0.8, 0.0], rtol=0, atol=1e-15)


def test_decay_is_logistic_of_minus_x():
    x = np.array([-40.0, -5.0, -2.0, -0.5, 0.0, 0.5, 2.0, 5.0, 40.0, 700.0])
    _, _, g = oracle.prologue(np.ones((1, 1, 1, 10)), np.ones((1, 1, 1, 10)), x.reshape(1, 1, 1, 10))
    alpha = np.exp(g.ravel())
    want = np.array([1.0 / (1.0 + math.exp(v)) if v < 700 else 0.0 for v in x])
    np.testing.assert_allclose(alpha, want, rtol=1e-13, atol=1e-300)
    assert g.ravel()[4] == -math.log(2.0)                 # softplus(0) = ln 2
    assert abs(g.ravel()[-1] + 700.0) < 1e-12               # softplus(x) -> x, no overflow
    assert np.all(g <= 0.0) and np.all(np.isfinite(g))


def test_prologue_then_forward_equals_forward_on_prepared_inputs():
    """The fused-prologue operator is the plain operator on the prologue's outputs."""
    rng = np.random.default_rng(22)
    B, T, H, dk, dv = 1, 9, 2, 4, 3
    q, k = rng.normal(size=(B, T, H, dk)), rng.normal(size=(B, T, H, dk))
    x = rng.normal(-2.0, 1.0, size=(B, T, H, dk))
    v = rng.normal(size=(B, T, H, dv))
    b = 1.0 / (1.0 + np.exp(-rng.normal(size=(B, T, H))))
    qn, kn, g = oracle.prologue(q, k, x)
    o1, s1 = oracle.forward(qn, kn, v, g, b)
    o2, s2 = oracle.forward(q / np.linalg.norm(q, axis=-1, keepdims=True),
                            k / np.linalg.norm(k, axis=-1, keepdims=True), v, -np.log1p(np.exp(x)), b)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(s1, s2, rtol=1e-12, atol=1e-13)


def test_rows_shorter_than_eps_are_divided_by_eps():
    """The floor of the divisor: a row of norm 1e-8 is divided by eps = 1e-6, so it
    keeps its direction with norm 1e-2 instead of being blown up to a unit vector."""
    q = np.zeros((1, 1, 1, 4))
    q[0, 0, 0] = [6e-9, 0.0, -8e-9, 0.0]
    qn, _, _ = oracle.prologue(q, q, np.zeros_like(q))
    np.testing.assert_allclose(qn[0, 0, 0], [6e-3, 0.0, -8e-3, 0.0], rtol=1e-12, atol=0)
    qn2, _, _ = oracle.prologue(q, q, np.zeros_like(q), eps=1e-9)
    np.testing.assert_allclose(qn2[0, 0, 0], [0.6, 0.0, -0.8, 0.0], rtol=1e-12, atol=0)
