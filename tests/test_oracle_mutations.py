"""Plant plausible mistakes in the oracle (on the CPU) and check that the pins
catch every one of them.  The mutations are compile-time-free switches of the
oracle's C code (flags >= 0x100); they are used by this file only."""
import numpy as np
import pytest

import oracle


def _inputs(seed, T=16, dk=8, dv=8):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((1, T, 1, dk))
    k = rng.standard_normal((1, T, 1, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((1, T, 1, dv))
    g = -rng.random((1, T, 1, dk))
    beta = rng.random((1, T, 1))
    S0 = 0.3 * rng.standard_normal((1, 1, dk, dv))
    return q, k, v, g, beta, S0


def pin_projection_form(flags):
    q, k, v, g, beta, S0 = _inputs(1)
    o, S = oracle.recurrent(q, k, v, g, beta, S0, flags=flags)
    St = S0[0, 0].copy()
    ok = True
    for t in range(q.shape[1]):
        kt = k[0, t, 0]
        St = (np.eye(len(kt)) - beta[0, t, 0] * np.outer(kt, kt)) @ np.diag(np.exp(g[0, t, 0])) @ St \
            + beta[0, t, 0] * np.outer(kt, v[0, t, 0])
        ok &= np.allclose(o[0, t, 0], St.T @ q[0, t, 0], rtol=1e-10, atol=1e-10)
    return bool(ok and np.allclose(S[0, 0], St, rtol=1e-10, atol=1e-10))


def pin_targeted_replacement(flags):
    q, k, v, g, beta, S0 = _inputs(2)
    beta[:] = 1.0
    _, _, hist = oracle.recurrent(q, k, v, g, beta, S0, flags=flags, return_history=True)
    return bool(np.allclose(np.einsum("btrcj,btrc->btrj", hist, k), v, atol=1e-10))


def pin_frozen_state(flags):
    q, k, v, g, beta, S0 = _inputs(3)
    g[:] = 0.0
    beta[:] = 0.0
    o, S = oracle.recurrent(q, k, v, g, beta, S0, flags=flags)
    ref = np.einsum("bhcj,bthc->bthj", S0, q)
    return bool(np.array_equal(S, S0) and np.allclose(o, ref, atol=1e-12))


def pin_onehot_gla(flags):
    rng = np.random.default_rng(4)
    T, dk, dv = 8, 8, 8
    perm = rng.permutation(dk)
    k = np.zeros((1, T, 1, dk))
    k[0, np.arange(T), 0, perm] = 1.0
    q = rng.standard_normal((1, T, 1, dk))
    v = rng.standard_normal((1, T, 1, dv))
    g = -rng.random((1, T, 1, dk))
    beta = rng.random((1, T, 1))
    o, _ = oracle.recurrent(q, k, v, g, beta, flags=flags)
    a = np.exp(g[0, :, 0])
    b = beta[0, :, 0]
    for t in range(T):
        ref = sum(b[j] * q[0, t, 0, perm[j]] * np.prod(a[j + 1: t + 1, perm[j]]) * v[0, j, 0]
                  for j in range(t + 1))
        if not np.allclose(o[0, t, 0], ref, atol=1e-10):
            return False
    return True


PINS = [pin_projection_form, pin_targeted_replacement, pin_frozen_state, pin_onehot_gla]


def test_all_pins_pass_unmutated():
    assert all(p(0) for p in PINS)


@pytest.mark.parametrize("mutation", [
    oracle.MUT_GATE_ON_VALUE_AXIS, oracle.MUT_PREDICT_UNDECAYED, oracle.MUT_OUTPUT_PRE_WRITE,
    oracle.MUT_NO_DECAY, oracle.MUT_READ_TRANSPOSED, oracle.MUT_ERROR_SIGN,
])
def test_each_mutation_is_caught(mutation):
    results = {p.__name__: p(mutation) for p in PINS}
    assert not all(results.values()), f"mutation {mutation:#x} slipped through: {results}"
