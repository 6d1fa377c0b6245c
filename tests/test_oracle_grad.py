"""Pins of the gradient oracle (oracle.grad.recurrent_grad and
gdn_recurrent_grad): central finite differences of the fp64 recurrences
themselves, a closed form for the gradient of a single step, consistency of
the forwards they differentiate with the pinned recurrences, and the chain
rules that tie the Gated DeltaNet gate's gradient to the per-channel one and
the raw projections' gradients to the prepared inputs' ones."""
import numpy as np

import oracle
from oracle.grad import gdn_recurrent_grad, recurrent_grad, recurrent_prep_grad


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


def _gdn_inputs(rng, B, T, H, dk, dv):
    q, k, v, g, beta, S0, do, dS = _inputs(rng, B, T, H, dk, dv)
    return q, k, v, g[..., 0].copy(), beta, S0, do, dS  # one gate per token and head


def _gdn_loss(q, k, v, g, beta, S0, do, dS):
    o, S = oracle.gdn_recurrent(q, k, v, g, beta, S0)
    return float((o * do).sum() + (S * dS).sum())


def test_gdn_forward_matches_the_pinned_gdn_recurrence():
    rng = np.random.default_rng(93)
    q, k, v, g, beta, S0, do, dS = _gdn_inputs(rng, 2, 9, 2, 5, 4)
    r = gdn_recurrent_grad(q, k, v, g, beta, S0, do, dS)
    o, S = oracle.gdn_recurrent(q, k, v, g, beta, S0)
    np.testing.assert_allclose(r["o"], o, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(r["S_T"], S, rtol=1e-12, atol=1e-13)


def test_gdn_gradients_match_central_differences():
    """Finite differences of the pinned Gated DeltaNet forward (oracle.gdn_recurrent)."""
    rng = np.random.default_rng(94)
    args = list(_gdn_inputs(rng, 1, 6, 2, 4, 3))
    r = gdn_recurrent_grad(*args)
    h = 1e-6
    for i, n in enumerate(["q", "k", "v", "g", "beta", "S0"]):
        x = args[i]
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            old = x[idx]
            x[idx] = old + h
            lp = _gdn_loss(*args)
            x[idx] = old - h
            lm = _gdn_loss(*args)
            x[idx] = old
            fd = (lp - lm) / (2 * h)
            assert abs(r["d" + n][idx] - fd) <= 1e-6 * max(1.0, abs(fd)), (n, idx, r["d" + n][idx], fd)


def test_gdn_gate_gradient_is_the_sum_over_channels():
    """Every key channel decays by the one g_t, so by the chain rule dL/dg_t is
    the per-channel gradient (of the same inputs with g repeated over dk)
    summed over the channels; the other gradients are the per-channel ones."""
    rng = np.random.default_rng(95)
    q, k, v, g, beta, S0, do, dS = _gdn_inputs(rng, 2, 7, 3, 5, 4)
    r = gdn_recurrent_grad(q, k, v, g, beta, S0, do, dS)
    g_full = np.repeat(g[..., None], q.shape[-1], axis=-1)
    rk = recurrent_grad(q, k, v, g_full, beta, S0, do, dS)
    np.testing.assert_allclose(r["dg"], rk["dg"].sum(-1), rtol=1e-11, atol=1e-12)
    for n in ("dq", "dk", "dv", "dbeta", "dS0"):
        np.testing.assert_allclose(r[n], rk[n], rtol=1e-11, atol=1e-12)


def _raw_inputs(rng, B, T, H, dk, dv):
    q = rng.standard_normal((B, T, H, dk)) * 2.0
    k = rng.standard_normal((B, T, H, dk)) * 0.5
    v = rng.standard_normal((B, T, H, dv))
    a = rng.standard_normal((B, T, H, dk)) - 1.0
    b = rng.standard_normal((B, T, H))
    S0 = rng.standard_normal((B, H, dk, dv)) * 0.3
    do = rng.standard_normal((B, T, H, dv))
    dS = rng.standard_normal((B, H, dk, dv))
    return q, k, v, a, b, S0, do, dS


def _prep_loss(q, k, v, a, b, S0, do, dS):
    o, S = oracle.recurrent_prep(q, k, v, a, b, S0)
    return float((o * do).sum() + (S * dS).sum())


def test_prep_forward_matches_the_pinned_prep_recurrence():
    rng = np.random.default_rng(96)
    q, k, v, a, b, S0, do, dS = _raw_inputs(rng, 2, 8, 2, 5, 4)
    r = recurrent_prep_grad(q, k, v, a, b, S0, do, dS)
    o, S = oracle.recurrent_prep(q, k, v, a, b, S0)
    np.testing.assert_allclose(r["o"], o, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(r["S_T"], S, rtol=1e-12, atol=1e-13)


def test_prep_gradients_match_central_differences():
    """Finite differences of the pinned forward from raw projections
    (oracle.recurrent_prep = oracle.prep then the recurrence)."""
    rng = np.random.default_rng(97)
    args = list(_raw_inputs(rng, 1, 5, 2, 4, 3))
    r = recurrent_prep_grad(*args)
    h = 1e-6
    for i, n in enumerate(["q", "k", "v", "a", "b", "S0"]):
        x = args[i]
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            old = x[idx]
            x[idx] = old + h
            lp = _prep_loss(*args)
            x[idx] = old - h
            lm = _prep_loss(*args)
            x[idx] = old
            fd = (lp - lm) / (2 * h)
            assert abs(r["d" + n][idx] - fd) <= 1e-6 * max(1.0, abs(fd)), (n, idx, r["d" + n][idx], fd)


def test_prep_gradients_are_the_prepared_ones_through_the_jacobians():
    """Closed forms of the preparation's derivatives applied to the gradient
    on the prepared inputs: for u = x / |x|, dx = (du - u (u . du)) / |x|;
    d(-softplus(a))/da = -sigmoid(a); d sigmoid(b)/db = beta (1 - beta)."""
    rng = np.random.default_rng(98)
    q, k, v, a, b, S0, do, dS = _raw_inputs(rng, 2, 6, 3, 5, 4)
    r = recurrent_prep_grad(q, k, v, a, b, S0, do, dS)
    qn, kn, g, beta = oracle.prep(q, k, a, b)
    rp = recurrent_grad(qn, kn, v, g, beta, S0, do, dS)
    for x, u, du, dx in ((q, qn, rp["dq"], r["dq"]), (k, kn, rp["dk"], r["dk"])):
        nrm = np.linalg.norm(x, axis=-1, keepdims=True)
        ref = (du - u * (u * du).sum(-1, keepdims=True)) / nrm
        np.testing.assert_allclose(dx, ref, rtol=1e-10, atol=1e-12)
    sig = 1.0 / (1.0 + np.exp(-a))
    np.testing.assert_allclose(r["da"], -sig * rp["dg"], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(r["db"], beta * (1 - beta) * rp["dbeta"], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(r["dv"], rp["dv"], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(r["dS0"], rp["dS0"], rtol=1e-10, atol=1e-12)
