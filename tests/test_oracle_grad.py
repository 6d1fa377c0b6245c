"""Pins of the gradient oracle (oracle.grad.recurrent_grad): central finite
differences of the fp64 recurrence itself, a closed form for the gradient of
a single step, and consistency of the forward it differentiates with the
pinned recurrence."""
import numpy as np

import oracle
from oracle.grad import recurrent_grad


def _inputs(rng, B, T, H, dk, dv):
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    g = -rng.random((B, T, H, dk)) * 0.7
    beta = rng.random((B, T, H))
    S0 = rng.standard_normal((B, H, dk, dv)) * 0.3
    do = rng.standard_normal((B, T, H, dv))
    dS = rng.standard_normal((B, H, dk, dv))
    return q, k, v, g, beta, S0, do, dS


def _loss(q, k, v, g, beta, S0, do, dS):
    o, S = oracle.recurrent(q, k, v, g, beta, S0)
    return float((o * do).sum() + (S * dS).sum())


def test_forward_matches_the_pinned_recurrence():
    rng = np.random.default_rng(90)
    q, k, v, g, beta, S0, do, dS = _inputs(rng, 2, 9, 2, 5, 4)
    r = recurrent_grad(q, k, v, g, beta, S0, do, dS)
    o, S = oracle.recurrent(q, k, v, g, beta, S0)
    np.testing.assert_allclose(r["o"], o, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(r["S_T"], S, rtol=1e-12, atol=1e-13)


def test_gradients_match_central_differences():
    rng = np.random.default_rng(91)
    args = list(_inputs(rng, 1, 6, 2, 4, 3))
    r = recurrent_grad(*args)
    names = ["q", "k", "v", "g", "beta", "S0"]
    h = 1e-6
    for i, n in enumerate(names):
        x = args[i]
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            old = x[idx]
            x[idx] = old + h
            lp = _loss(*args)
            x[idx] = old - h
            lm = _loss(*args)
            x[idx] = old
            fd = (lp - lm) / (2 * h)
            assert abs(r["d" + n][idx] - fd) <= 1e-6 * max(1.0, abs(fd)), (n, idx, r["d" + n][idx], fd)


def test_single_step_closed_form():
    """T = 1 from S0: o = (D S0 + k e^T)^T q with e = beta (v - (D S0)^T k), so
    d o_j / d v_j' = beta (k . q) [j == j'] and dS0 = D (q do^T - beta k ((k.q) do)^T)."""
    rng = np.random.default_rng(92)
    q, k, v, g, beta, S0, do, _ = _inputs(rng, 1, 1, 1, 5, 4)
    r = recurrent_grad(q, k, v, g, beta, S0, do, None)
    kq = float(k[0, 0, 0] @ q[0, 0, 0])
    b = beta[0, 0, 0]
    np.testing.assert_allclose(r["dv"][0, 0, 0], b * kq * do[0, 0, 0], rtol=1e-12)
    D = np.exp(g[0, 0, 0])
    ref = D[:, None] * (np.outer(q[0, 0, 0], do[0, 0, 0]) - b * kq * np.outer(k[0, 0, 0], do[0, 0, 0]))
    np.testing.assert_allclose(r["dS0"][0, 0], ref, rtol=1e-12, atol=1e-14)
