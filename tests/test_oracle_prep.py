"""Pins of the oracle's input preparation (oracle.prep) against closed forms
and invariants of its three maps: L2 normalisation of q and k, log alpha =
-softplus(a), beta = sigmoid(b)."""
import math

import numpy as np

import oracle


def test_rows_have_unit_norm_and_zero_rows_stay_zero():
    rng = np.random.default_rng(50)
    q = rng.standard_normal((2, 5, 3, 16)) * 7.0
    k = rng.standard_normal((2, 5, 3, 16)) * 0.01
    k[1, 2, 0] = 0.0
    qn, kn, _, _ = oracle.prep(q, k, np.zeros(1), np.zeros(1))
    np.testing.assert_allclose(np.linalg.norm(qn, axis=-1), 1.0, rtol=0, atol=1e-14)
    mask = np.ones(k.shape[:-1], bool)
    mask[1, 2, 0] = False
    np.testing.assert_allclose(np.linalg.norm(kn, axis=-1)[mask], 1.0, rtol=0, atol=1e-14)
    assert np.all(kn[1, 2, 0] == 0.0)


def test_normalisation_is_scale_invariant_and_idempotent():
    rng = np.random.default_rng(51)
    q = rng.standard_normal((1, 4, 2, 8))
    c = np.array([3.0, 0.25, 1e3, 1e-3]).reshape(1, 4, 1, 1)
    q1, _, _, _ = oracle.prep(q, q, np.zeros(1), np.zeros(1))
    q2, _, _, _ = oracle.prep(q * c, q, np.zeros(1), np.zeros(1))
    np.testing.assert_allclose(q1, q2, rtol=1e-14, atol=1e-15)
    q3, _, _, _ = oracle.prep(q1, q1, np.zeros(1), np.zeros(1))
    np.testing.assert_allclose(q3, q1, rtol=1e-15, atol=1e-16)
    # direction is kept: q1 is a positive multiple of q
    ratio = q1 / q
    np.testing.assert_allclose(ratio, ratio[..., :1] * np.ones_like(ratio), rtol=1e-13)
    assert np.all(ratio > 0)


def test_gate_activation_special_values_and_asymptotes():
    a = np.array([0.0, 50.0, -50.0, 1.0, -1.0, 700.0, -700.0])
    _, _, g, _ = oracle.prep(np.ones(4), np.ones(4), a, np.zeros(1))
    assert abs(g[0] + math.log(2.0)) < 1e-16
    assert abs(g[1] + 50.0) < 1e-13                      # softplus(a) -> a
    assert abs(g[2] + math.exp(-50.0)) < 1e-30           # softplus(a) -> e^a
    assert np.isfinite(g).all() and g[5] == -700.0 and -1e-300 < g[6] <= 0.0
    # alpha = e^g is the logistic function of -a: 1 / (1 + e^a)
    aa = np.linspace(-30, 30, 61)
    _, _, gg, _ = oracle.prep(np.ones(4), np.ones(4), aa, np.zeros(1))
    np.testing.assert_allclose(np.exp(gg), 1.0 / (1.0 + np.exp(aa)), rtol=1e-13)
    # softplus(a) - softplus(-a) = a
    _, _, gn, _ = oracle.prep(np.ones(4), np.ones(4), -aa, np.zeros(1))
    np.testing.assert_allclose(-gg + gn, aa, rtol=0, atol=1e-13)


def test_beta_is_the_logistic_function():
    b = np.array([0.0, 3.0, -3.0, 40.0, -40.0, 800.0, -800.0])
    _, _, _, beta = oracle.prep(np.ones(4), np.ones(4), np.zeros(1), b)
    assert beta[0] == 0.5
    np.testing.assert_allclose(beta[1], 1.0 / (1.0 + math.exp(-3.0)), rtol=1e-15)
    np.testing.assert_allclose(beta[1] + beta[2], 1.0, rtol=0, atol=1e-15)  # symmetry
    assert beta[5] == 1.0 and beta[6] == 0.0 and np.all((beta >= 0) & (beta <= 1))


def test_recurrent_prep_equals_recurrent_on_prepared_inputs():
    rng = np.random.default_rng(52)
    q = rng.standard_normal((1, 12, 2, 6))
    k = rng.standard_normal((1, 12, 2, 6))
    v = rng.standard_normal((1, 12, 2, 5))
    a = rng.standard_normal((1, 12, 2, 6))
    b = rng.standard_normal((1, 12, 2))
    o1, S1 = oracle.recurrent_prep(q, k, v, a, b)
    qn = q / np.linalg.norm(q, axis=-1, keepdims=True)
    kn = k / np.linalg.norm(k, axis=-1, keepdims=True)
    o2, S2 = oracle.recurrent(qn, kn, v, -np.log1p(np.exp(a)), 1.0 / (1.0 + np.exp(-b)))
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(S1, S2, rtol=1e-12, atol=1e-13)
