"""Gradients of the KDA recurrence, in fp64 on the CPU, for checking the
backward kernels.  TEST INFRASTRUCTURE ONLY (same rule as the rest of this
package: only tests/, the smoke check and the benchmark's CPU baseline use it).

The forward map is the token-by-token definition ("Kimi K3 notes 1: KDA"
sections 4-5; "Deriving Kimi Delta Attention from scratch" sections 3-5),
written out with plain PyTorch fp64 CPU tensor ops:
    S~ = Diag(e^{g_t}) S;  v^ = S~^T k_t;  e = beta_t (v_t - v^);
    S = S~ + k_t e^T;      o_t = S^T q_t,
and the gradients are reverse-mode automatic differentiation of that loop
(torch.autograd), i.e. the exact derivative of the defined function up to
fp64 rounding.  The pages leave the backward pass to the reader ("Deriving
KDA from scratch" section 6 names the chunked mode only for the forward);
nothing here depends on a particular backward algorithm.
"""
from __future__ import annotations

import numpy as np
import torch


def recurrent_grad(q, k, v, g, beta, S0, do, dS_T=None):
    """For one batch of independent sequences (no packing): q, k, g [B,T,H,dk];
    v, do [B,T,H,dv]; beta [B,T,H]; S0 [B,H,dk,dv] or None; dS_T (gradient of
    the final state) [B,H,dk,dv] or None.  Returns a dict of float64 numpy
    arrays dq, dk, dv, dg, dbeta, dS0 (dS0 is None when S0 is None) and the
    forward o, S_T."""
    return _grad(q, k, v, g, beta, S0, do, dS_T, scalar_gate=False)


def gdn_recurrent_grad(q, k, v, g, beta, S0, do, dS_T=None):
    """Gated DeltaNet: one decay per token and head ("Kimi K3 notes 1: KDA"
    section 3; "Linear / sparse attention" tutorial section 5.2), g [B,T,H],
    so the loop decays the whole state by the scalar e^{g_t}:
        S~ = e^{g_t} S;  then the same delta-rule write and read.
    Arguments and result as recurrent_grad, with dg [B,T,H]."""
    return _grad(q, k, v, g, beta, S0, do, dS_T, scalar_gate=True)


def recurrent_prep_grad(q, k, v, a, b, S0, do, dS_T=None):
    """The recurrence fed by the input preparation of oracle.prep (q, k
    L2-normalised with the norm clamped at 1e-12, log alpha = -softplus(a),
    beta = sigmoid(b); "Kimi K3 notes 1: KDA" section 4, "Linear / sparse
    attention" tutorial section 10), differentiated with respect to the RAW
    q, k, a [B,T,H,dk] and b [B,T,H].  Returns the dict of recurrent_grad with
    dq, dk, da, db (gradients of the raw inputs) in place of dq, dk, dg, dbeta."""
    return _grad(q, k, v, a, b, S0, do, dS_T, scalar_gate=False, prep=True)


def _grad(q, k, v, g, beta, S0, do, dS_T, scalar_gate, prep=False):
    t64 = lambda x: torch.as_tensor(np.asarray(x if not hasattr(x, "detach") else x.detach().cpu(),
                                               dtype=np.float64)).clone()
    q, k, v, g, beta = (t64(x).requires_grad_(True) for x in (q, k, v, g, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if g.shape != ((B, T, H) if scalar_gate else (B, T, H, dk)):
        raise ValueError("g must be [B,T,H] for a scalar gate and [B,T,H,dk] otherwise")
    S = (t64(S0) if S0 is not None else torch.zeros(B, H, dk, dv, dtype=torch.float64)).requires_grad_(S0 is not None)
    S_init = S
    qr, kr, ar, br = q, k, g, beta  # the leaves
    if prep:  # raw projections: the preparation first, in the leaves' graph
        q = q / q.norm(dim=-1, keepdim=True).clamp_min(1e-12)
        k = k / k.norm(dim=-1, keepdim=True).clamp_min(1e-12)
        g = -torch.logaddexp(torch.zeros_like(g), g)
        beta = torch.sigmoid(beta)
    outs = []
    for t in range(T):
        a = torch.exp(g[:, t])                                # [B,H] or [B,H,dk]
        St = (a[..., None, None] if scalar_gate else a.unsqueeze(-1)) * S  # S~
        vh = torch.einsum("bhcj,bhc->bhj", St, k[:, t])
        e = beta[:, t].unsqueeze(-1) * (v[:, t] - vh)
        S = St + k[:, t].unsqueeze(-1) * e.unsqueeze(-2)
        outs.append(torch.einsum("bhcj,bhc->bhj", S, q[:, t]))
    o = torch.stack(outs, 1)
    loss = (o * t64(do)).sum()
    if dS_T is not None:
        loss = loss + (S * t64(dS_T)).sum()
    leaves = [qr, kr, v, ar, br] + ([S_init] if S0 is not None else [])
    grads = torch.autograd.grad(loss, leaves)
    names = ("dq", "dk", "dv", "da", "db") if prep else ("dq", "dk", "dv", "dg", "dbeta")
    res = {n: x.numpy() for n, x in zip(names, grads[:5])}
    res["dS0"] = grads[5].numpy() if S0 is not None else None
    res["o"] = o.detach().numpy()
    res["S_T"] = S.detach().numpy()
    return res
