"""Helpers for the GPU parity tests: run the fp64 oracle on selected
(sequence, head) units of a workload and compare with the CUDA results using
the max-over-slices relative RMS error."""
from __future__ import annotations

import json
import os

import numpy as np
import torch

import oracle

TOL = {torch.bfloat16: 1e-2, torch.float32: 1e-4}


def record_margin(worst_o, worst_S, tol, units):
    """Appends the worst errors of one comparison to the JSON-lines file named
    by the environment variable KDA_PARITY_LOG (when it is set), so that the
    margin under each tolerance is on record, not only pass or fail."""
    path = os.environ.get("KDA_PARITY_LOG")
    if not path:
        return
    test = os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0]
    with open(path, "a") as f:
        f.write(json.dumps({"test": test, "worst_o": float(worst_o), "worst_S": float(worst_S), "tol": tol,
                            "units": int(units)}) + "\n")


def seq_bounds(inp, n):
    cu = inp.get("cu_seqlens")
    if cu is not None:
        cu = cu.cpu().tolist()
        return 0, cu[n], cu[n + 1]
    T = inp["q"].shape[1]
    return n, 0, T


def gather_units(inp, units, names=("q", "k", "v", "g", "beta")):
    """Pack the selected units into a [1, sumT, 1, d] layout with cu_seqlens."""
    cols = {n: [] for n in names}
    S0 = []
    cu = [0]
    for (n, h) in units:
        b, t0, t1 = seq_bounds(inp, n)
        for name in cols:
            x = inp[name]
            cols[name].append(x[b, t0:t1, h].detach().cpu().double())
        cu.append(cu[-1] + (t1 - t0))
        if inp.get("S0") is not None:
            S0.append(inp["S0"][n, h].detach().cpu().double())
    packed = {}
    for name, parts in cols.items():
        cat = torch.cat(parts, 0) if parts else torch.zeros(0)
        packed[name] = (cat.unsqueeze(0).unsqueeze(2).numpy() if name not in ("beta", "b")
                        else cat.reshape(1, -1, 1).numpy())
    S0 = torch.stack(S0).unsqueeze(1).numpy() if S0 else None
    return packed, S0, np.array(cu, dtype=np.int64)


def oracle_units(inp, units):
    """fp64 oracle outputs for ``units``: list of (o [T_n, dv], S [dk, dv])."""
    p, S0, cu = gather_units(inp, units)
    if inp["g"].dim() == 3:  # Gated DeltaNet: one gate per token and head
        o, S = oracle.gdn_recurrent(p["q"], p["k"], p["v"], p["g"], p["beta"], S0, cu_seqlens=cu)
    else:
        o, S = oracle.recurrent(p["q"], p["k"], p["v"], p["g"], p["beta"], S0, cu_seqlens=cu)
    return [(o[0, cu[i]:cu[i + 1], 0], S[i, 0]) for i in range(len(units))]


def compare_units_prep(inp, o_gpu, S_gpu, units, tol):
    """compare_units for raw projections (q, k, v, a, b): the oracle prepares
    the selected units in fp64, then runs the recurrence."""
    p, S0, cu = gather_units(inp, units, names=("q", "k", "v", "a", "b"))
    o, S = oracle.recurrent_prep(p["q"], p["k"], p["v"], p["a"], p["b"], S0, cu_seqlens=cu)
    worst_o = worst_S = 0.0
    for i, (n, h) in enumerate(units):
        b, t0, t1 = seq_bounds(inp, n)
        if t1 > t0:
            worst_o = max(worst_o, rel_rms(o_gpu[b, t0:t1, h].float().cpu().numpy(), o[0, cu[i]:cu[i + 1], 0]))
        worst_S = max(worst_S, rel_rms(S_gpu[n, h].cpu().numpy(), S[i, 0]))
    record_margin(worst_o, worst_S, tol, len(units))
    assert np.isfinite(worst_o) and np.isfinite(worst_S)
    assert worst_o <= tol, f"o rel-RMS {worst_o:.3e} > {tol}"
    assert worst_S <= tol, f"S rel-RMS {worst_S:.3e} > {tol}"
    return worst_o, worst_S


def rel_rms(x, ref):
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    num = np.sqrt(((x - ref) ** 2).sum())
    den = np.sqrt((ref ** 2).sum())
    if den < 1e-30:
        return num / np.sqrt(max(x.size, 1))
    return num / den


def compare_units(inp, o_gpu, S_gpu, units, tol):
    """Max rel-RMS error over units of o (over T x dv) and S_final."""
    refs = oracle_units(inp, units)
    worst_o = worst_S = 0.0
    for (n, h), (o_ref, S_ref) in zip(units, refs):
        b, t0, t1 = seq_bounds(inp, n)
        og = o_gpu[b, t0:t1, h].float().cpu().numpy()
        if t1 > t0:
            worst_o = max(worst_o, rel_rms(og, o_ref))
        if S_gpu is not None:
            worst_S = max(worst_S, rel_rms(S_gpu[n, h].cpu().numpy(), S_ref))
    record_margin(worst_o, worst_S, tol, len(units))
    assert np.isfinite(worst_o) and np.isfinite(worst_S)
    assert worst_o <= tol, f"o rel-RMS {worst_o:.3e} > {tol}"
    assert worst_S <= tol, f"S rel-RMS {worst_S:.3e} > {tol}"
    return worst_o, worst_S


def sample_units(N, H, count, seed, must=()):
    rng = np.random.default_rng(seed)
    units = set(tuple(u) for u in must)
    all_units = N * H
    while len(units) < min(count, all_units):
        u = int(rng.integers(all_units))
        units.add((u // H, u % H))
    return sorted(units)
