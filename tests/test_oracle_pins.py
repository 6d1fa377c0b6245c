"""Pins for the fp64 oracle, against what the pages and the mathematics fix.

None of these re-types the oracle's own loop: each compares it with a
different formula (a closed form, the page's projection form, a quadratic
masked form, exact rational arithmetic) or with an invariant the pages state.
The companion file test_oracle_mutations.py plants mistakes in the oracle and
checks that at least one of these pins fails for each.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden", "page5_appendixA.json")


def rand_inputs(rng, B, T, H, dk, dv, g_scale=0.3, unit_keys=True, s0=0.1):
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    if unit_keys:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    g = -g_scale * rng.random((B, T, H, dk)) * 2.0
    beta = rng.random((B, T, H))
    S0 = s0 * rng.standard_normal((B, H, dk, dv)) if s0 else None
    return q, k, v, g, beta, S0


def causal_linear_attention(q, k, v):
    """Quadratic masked form o = ((Q K^T) o M) V ("Linear / sparse attention"
    tutorial, section 2.2 table, parallel view; section 6.2 intra term)."""
    T = q.shape[0]
    M = np.tril(np.ones((T, T)))
    return ((q @ k.T) * M) @ v


# ---- pin 1: frozen state (beta = 0, alpha = 1) --------------------------------
def test_frozen_state_beta0_alpha1():
    rng = np.random.default_rng(1)
    q, k, v, g, beta, S0 = rand_inputs(rng, 2, 9, 3, 8, 5)
    g[:] = 0.0
    beta[:] = 0.0
    o, S = oracle.recurrent(q, k, v, g, beta, S0)
    np.testing.assert_array_equal(S, S0)
    # o_t = S0^T q_t for every token
    ref = np.einsum("bhcj,bthc->bthj", S0, q)
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-14)


# ---- pin 2: orthonormal keys, alpha = beta = 1: causal linear attention ------
def test_orthonormal_keys_reduce_to_linear_attention():
    rng = np.random.default_rng(2)
    T = d = 32
    Qm, _ = np.linalg.qr(rng.standard_normal((d, d)))
    keys = Qm.T[:T]  # rows are orthonormal
    q = rng.standard_normal((1, T, 1, d))
    v = rng.standard_normal((1, T, 1, d))
    k = keys.reshape(1, T, 1, d)
    g = np.zeros((1, T, 1, d))
    beta = np.ones((1, T, 1))
    o, S = oracle.recurrent(q, k, v, g, beta)
    ref = causal_linear_attention(q[0, :, 0], keys, v[0, :, 0])
    np.testing.assert_allclose(o[0, :, 0], ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(S[0, 0], keys.T @ v[0, :, 0], rtol=0, atol=1e-12)


# ---- pin 3: erase term dropped, beta = 1: additive linear attention ----------
def test_erase_dropped_is_additive_for_any_keys():
    gold = json.load(open(GOLD))["erase_term_dropped_equals_additive"]
    rng = np.random.default_rng(3)
    T, d = gold["L"], gold["d"]
    q = rng.standard_normal((1, T, 1, d))
    k = rng.standard_normal((1, T, 1, d))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((1, T, 1, d))
    g = np.zeros((1, T, 1, d))
    beta = np.ones((1, T, 1))
    o, S = oracle.recurrent(q, k, v, g, beta, flags=oracle.NO_ERASE)
    # additive state, accumulated in the same order: the page prints |diff| = 0
    S_add = np.zeros((d, d))
    for t in range(T):
        S_add = S_add + np.outer(k[0, t, 0], v[0, t, 0])
    assert np.abs(S[0, 0] - S_add).max() == gold["printed_abs_diff"]
    ref = causal_linear_attention(q[0, :, 0], k[0, :, 0], v[0, :, 0])
    np.testing.assert_allclose(o[0, :, 0], ref, rtol=0, atol=1e-12)
    # ... and with the erase term kept, non-orthogonal keys give a difference
    _, S_delta = oracle.recurrent(q, k, v, g, beta)
    assert np.linalg.norm(S_delta[0, 0] - S_add) > 1e-2


# ---- pin 4: GLA closed form for one-hot distinct keys ------------------------
@pytest.mark.parametrize("with_s0", [False, True])
def test_onehot_keys_gated_closed_form(with_s0):
    rng = np.random.default_rng(4)
    T, dk, dv = 10, 12, 6
    perm = rng.permutation(dk)[:T]
    k = np.zeros((1, T, 1, dk))
    k[0, np.arange(T), 0, perm] = 1.0
    q = rng.standard_normal((1, T, 1, dk))
    v = rng.standard_normal((1, T, 1, dv))
    g = -rng.random((1, T, 1, dk))
    beta = rng.random((1, T, 1))
    S0 = rng.standard_normal((1, 1, dk, dv)) if with_s0 else None
    o, S = oracle.recurrent(q, k, v, g, beta, S0)
    a = np.exp(g[0, :, 0])  # alpha[t, c]
    b = beta[0, :, 0]
    # row c of the state evolves on its own; decay D(c, i..t) = prod alpha
    s0 = S0[0, 0] if with_s0 else np.zeros((dk, dv))
    rows = np.zeros((T + 1, dk, dv))
    cur = s0.copy()
    written = {}
    for t in range(T):
        cur = cur * a[t][:, None]                       # decay every row
        c = perm[t]
        cur[c] = cur[c] + b[t] * (v[0, t, 0] - cur[c])  # replace along e_c
        rows[t + 1] = cur
        written[c] = t
    # closed form for the output: sum over written rows + decayed initial rows
    for t in range(T):
        ref = np.zeros(dv)
        for c in range(dk):
            dec0 = np.prod(a[: t + 1, c])
            if c in perm[: t + 1]:
                j = int(np.where(perm == c)[0][0])
                dec_after = np.prod(a[j + 1: t + 1, c])
                dec_before = np.prod(a[: j + 1, c])
                val = dec_after * ((1 - b[j]) * dec_before * s0[c] + b[j] * v[0, j, 0])
            else:
                val = dec0 * s0[c]
            ref += q[0, t, 0, c] * val
        np.testing.assert_allclose(o[0, t, 0], ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S[0, 0], rows[T], rtol=1e-12, atol=1e-12)
    if not with_s0:
        # pure GLA form: o_t = sum_{j<=t} beta_j q_{t,pi(j)} prod_{i=j+1..t} alpha_{i,pi(j)} v_j
        for t in range(T):
            ref = sum(b[j] * q[0, t, 0, perm[j]] * np.prod(a[j + 1: t + 1, perm[j]]) * v[0, j, 0]
                      for j in range(t + 1))
            np.testing.assert_allclose(o[0, t, 0], ref, rtol=1e-12, atol=1e-12)


# ---- pin 5: targeted replacement (beta = 1, unit keys) -----------------------
def test_targeted_replacement_reads_back_value():
    rng = np.random.default_rng(5)
    q, k, v, g, beta, S0 = rand_inputs(rng, 2, 20, 2, 16, 8)
    beta[:] = 1.0
    o, S, hist = oracle.recurrent(q, k, v, g, beta, S0, return_history=True)
    readback = np.einsum("btrcj,btrc->btrj", hist, k)
    np.testing.assert_allclose(readback, v, rtol=0, atol=1e-12)


# ---- pin 6: scalar gate = Gated DeltaNet, alpha = 1 = DeltaNet ---------------
def _gated_deltanet_value_by_key(k, v, q, alpha, beta, M0):
    """Page 5 section 5.2 convention: state M is dv x dk,
    M_t = alpha_t M_{t-1} (I - beta_t k k^T) + beta_t v k^T, o_t = M_t q_t."""
    T, dk = k.shape
    M = M0.copy()
    out = []
    eye = np.eye(dk)
    for t in range(T):
        M = alpha[t] * M @ (eye - beta[t] * np.outer(k[t], k[t])) + beta[t] * np.outer(v[t], k[t])
        out.append(M @ q[t])
    return np.array(out), M


@pytest.mark.parametrize("scalar_gate", [True, False])
def test_scalar_gate_matches_gated_deltanet(scalar_gate):
    rng = np.random.default_rng(6)
    T, dk, dv = 24, 10, 7
    q, k, v, g, beta, S0 = rand_inputs(rng, 1, T, 1, dk, dv)
    if scalar_gate:
        gs = -rng.random(T)
        g[0, :, 0, :] = gs[:, None]
        alpha = np.exp(gs)
    else:  # DeltaNet: alpha = 1 (page 5 section 5.1 boxed update)
        g[:] = 0.0
        alpha = np.ones(T)
    o, S = oracle.recurrent(q, k, v, g, beta, S0)
    ref_o, ref_M = _gated_deltanet_value_by_key(k[0, :, 0], v[0, :, 0], q[0, :, 0], alpha,
                                                beta[0, :, 0], S0[0, 0].T)
    np.testing.assert_allclose(o[0, :, 0], ref_o, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S[0, 0], ref_M.T, rtol=1e-12, atol=1e-12)


def test_gdn_oracle_matches_gated_deltanet():
    """oracle.gdn_recurrent (gate [B,T,H]) against the tutorial's Gated
    DeltaNet update, per (sequence, head), two heads with different gates."""
    rng = np.random.default_rng(16)
    T, dk, dv, H = 20, 9, 5, 2
    q, k, v, g, beta, S0 = rand_inputs(rng, 1, T, H, dk, dv)
    gs = -rng.random((1, T, H)) * 2.0
    o, S = oracle.gdn_recurrent(q, k, v, gs, beta, S0)
    for h in range(H):
        ref_o, ref_M = _gated_deltanet_value_by_key(k[0, :, h], v[0, :, h], q[0, :, h],
                                                    np.exp(gs[0, :, h]), beta[0, :, h], S0[0, h].T)
        np.testing.assert_allclose(o[0, :, h], ref_o, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(S[0, h], ref_M.T, rtol=1e-12, atol=1e-12)


# ---- pin 7: the projection form of "Kimi K3 notes 1", section 4 ---------------
def test_projection_form():
    """S_t = (I - beta k k^T) Diag(alpha_t) S_{t-1} + beta k v^T, o_t = S_t^T q_t."""
    rng = np.random.default_rng(7)
    T, dk, dv = 30, 9, 11
    q, k, v, g, beta, S0 = rand_inputs(rng, 1, T, 1, dk, dv, g_scale=1.0)
    o, S = oracle.recurrent(q, k, v, g, beta, S0)
    St = S0[0, 0].copy()
    eye = np.eye(dk)
    for t in range(T):
        kt = k[0, t, 0]
        St = (eye - beta[0, t, 0] * np.outer(kt, kt)) @ np.diag(np.exp(g[0, t, 0])) @ St \
            + beta[0, t, 0] * np.outer(kt, v[0, t, 0])
        np.testing.assert_allclose(o[0, t, 0], St.T @ q[0, t, 0], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S[0, 0], St, rtol=1e-12, atol=1e-12)


def test_exact_rational_tiny_example():
    """Exact rational arithmetic on dyadic inputs: alpha in {1/2, 1/4, 3/4, 1}."""
    alpha = [[Fraction(1, 2), Fraction(3, 4)], [Fraction(1, 4), Fraction(1)], [Fraction(3, 4), Fraction(1, 2)]]
    kk = [[Fraction(1), Fraction(0)], [Fraction(3, 5), Fraction(4, 5)], [Fraction(0), Fraction(1)]]
    vv = [[Fraction(2), Fraction(-1), Fraction(1, 2)], [Fraction(1), Fraction(1), Fraction(-3)],
          [Fraction(-1, 2), Fraction(5, 4), Fraction(1)]]
    qq = [[Fraction(1, 2), Fraction(-1)], [Fraction(1), Fraction(1, 4)], [Fraction(-3, 4), Fraction(2)]]
    bb = [Fraction(1, 2), Fraction(1, 4), Fraction(1)]
    S = [[Fraction(1, 8), Fraction(0), Fraction(-1, 4)], [Fraction(1, 2), Fraction(1, 16), Fraction(0)]]
    S0 = np.array([[float(x) for x in row] for row in S])
    outs = []
    for t in range(3):
        St = [[alpha[t][c] * S[c][j] for j in range(3)] for c in range(2)]
        vhat = [sum(St[c][j] * kk[t][c] for c in range(2)) for j in range(3)]
        e = [bb[t] * (vv[t][j] - vhat[j]) for j in range(3)]
        S = [[St[c][j] + kk[t][c] * e[j] for j in range(3)] for c in range(2)]
        outs.append([sum(S[c][j] * qq[t][c] for c in range(2)) for j in range(3)])
    f = lambda m: np.array([[float(x) for x in r] for r in m])
    q = f(qq).reshape(1, 3, 1, 2)
    k = f(kk).reshape(1, 3, 1, 2)
    v = f(vv).reshape(1, 3, 1, 3)
    g = np.log(f(alpha)).reshape(1, 3, 1, 2)
    beta = np.array([float(x) for x in bb]).reshape(1, 3, 1)
    o, Sf = oracle.recurrent(q, k, v, g, beta, S0.reshape(1, 1, 2, 3))
    np.testing.assert_allclose(o[0, :, 0], f(outs), rtol=0, atol=1e-14)
    np.testing.assert_allclose(Sf[0, 0], f(S), rtol=0, atol=1e-14)


# ---- pin 8: schedule equivalence (chunk == recurrent) -------------------------
def test_chunk_equals_recurrent_page5_chunk_sizes():
    gold = json.load(open(GOLD))["schedule_equivalence"]
    rng = np.random.default_rng(8)
    T = gold["L"]
    q, k, v, g, beta, S0 = rand_inputs(rng, 1, T, 2, 6, 6, g_scale=1.0)
    o, S = oracle.recurrent(q, k, v, g, beta, S0)
    for C in gold["chunk_sizes"]:
        oc, Sc = oracle.chunk(q, k, v, g, beta, S0, chunk_size=C)
        assert np.abs(oc - o).max() < gold["atol_printed_fp32"]
        assert oracle.rel_rms_per_slice(oc, o) < 1e-12
        assert oracle.rel_rms_per_slice(Sc, S) < 1e-12


@pytest.mark.parametrize("C", [1, 4, 7, 16, 64, 100])
def test_chunk_equals_recurrent(C):
    rng = np.random.default_rng(9)
    T = 100
    q, k, v, g, beta, S0 = rand_inputs(rng, 2, T, 2, 16, 12, g_scale=2.0)
    o, S = oracle.recurrent(q, k, v, g, beta, S0)
    oc, Sc = oracle.chunk(q, k, v, g, beta, S0, chunk_size=C)
    assert oracle.rel_rms_per_slice(oc, o) < 1e-12
    assert oracle.rel_rms_per_slice(Sc, S) < 1e-12


def test_chunk_strong_decay_no_overflow():
    # fast-forgetting channels: cumulative log-decay far below -88 inside a chunk
    rng = np.random.default_rng(10)
    q, k, v, g, beta, S0 = rand_inputs(rng, 1, 64, 1, 8, 8)
    g[..., :3] = -12.0
    o, S = oracle.recurrent(q, k, v, g, beta, S0)
    oc, Sc = oracle.chunk(q, k, v, g, beta, S0, chunk_size=64)
    assert np.isfinite(oc).all() and np.isfinite(Sc).all()
    assert oracle.rel_rms_per_slice(oc, o) < 1e-12


# ---- pin 9: split invariance and decode == prefill ----------------------------
def test_split_invariance_and_decode_steps():
    rng = np.random.default_rng(11)
    T1, T2 = 13, 22
    q, k, v, g, beta, S0 = rand_inputs(rng, 2, T1 + T2, 3, 8, 8)
    o, S = oracle.recurrent(q, k, v, g, beta, S0)
    sl1 = (slice(None), slice(0, T1))
    sl2 = (slice(None), slice(T1, None))
    o1, S1 = oracle.recurrent(q[sl1], k[sl1], v[sl1], g[sl1], beta[sl1], S0)
    o2, S2 = oracle.recurrent(q[sl2], k[sl2], v[sl2], g[sl2], beta[sl2], S1)
    np.testing.assert_allclose(np.concatenate([o1, o2], axis=1), o, rtol=0, atol=1e-13)
    np.testing.assert_allclose(S2, S, rtol=0, atol=1e-13)
    # T single-token steps, state carried
    St = S0
    for t in range(T1 + T2):
        s = (slice(None), slice(t, t + 1))
        ot, St = oracle.recurrent(q[s], k[s], v[s], g[s], beta[s], St)
        np.testing.assert_allclose(ot[:, 0], o[:, t], rtol=0, atol=1e-13)
    np.testing.assert_allclose(St, S, rtol=0, atol=1e-13)


# ---- pin 10: packed varlen == separate calls ----------------------------------
def test_varlen_equals_separate():
    rng = np.random.default_rng(12)
    lens = [5, 1, 17, 0, 9]
    Ttot = sum(lens)
    q, k, v, g, beta, _ = rand_inputs(rng, 1, Ttot, 2, 8, 4)
    S0 = rng.standard_normal((len(lens), 2, 8, 4))
    cu = np.cumsum([0] + lens)
    o, S = oracle.recurrent(q, k, v, g, beta, S0, cu_seqlens=cu)
    oc, Sc = oracle.chunk(q, k, v, g, beta, S0, cu_seqlens=cu, chunk_size=4)
    for n, L in enumerate(lens):
        s = (slice(None), slice(cu[n], cu[n + 1]))
        on, Sn = oracle.recurrent(q[s], k[s], v[s], g[s], beta[s], S0[n:n + 1])
        np.testing.assert_allclose(o[:, cu[n]:cu[n + 1]], on, rtol=0, atol=1e-13)
        np.testing.assert_allclose(S[n], Sn[0], rtol=0, atol=1e-13)
        if L == 0:
            np.testing.assert_array_equal(S[n], S0[n])
    assert oracle.rel_rms_per_slice(Sc, S) < 1e-12
    np.testing.assert_allclose(oc, o, rtol=0, atol=1e-12)


# ---- pin 11: state shape independent of T -------------------------------------
def test_state_shape_independent_of_length():
    gold = json.load(open(GOLD))["state_shape"]
    rng = np.random.default_rng(13)
    shapes = set()
    for T in range(1, gold["L"] + 1):
        q, k, v, g, beta, S0 = rand_inputs(rng, 1, T, 1, gold["d"], gold["d"])
        _, S = oracle.recurrent(q, k, v, g, beta, S0)
        shapes.add(S.shape[2:])
    assert shapes == {(gold["d"], gold["d"])}


def test_tolerance_metric():
    ref = np.ones((1, 4, 2, 3))
    x = ref.copy()
    x[0, :, 1, :] *= 1.01
    assert abs(oracle.rel_rms_per_slice(x, ref) - 0.01) < 1e-12
    z = np.zeros((2, 2, 3, 3))
    assert oracle.rel_rms_per_slice(z, z) == 0.0
