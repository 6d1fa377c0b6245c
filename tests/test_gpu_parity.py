"""GPU parity: the CUDA path (called through the C ABI via the Python
binding) against the fp64 oracle on the same seeded inputs.

Tolerance: max over (sequence, head) slices of the relative RMS error of o
(over T x dv) and of the final state, 1e-2 for bf16 q/k/v and 1e-4 for fp32.
"""
import numpy as np
import pytest
import torch

import kimi_delta_attention_31_b200 as kda
import kda_workloads as W
import oracle
from parity_util import TOL, compare_units, oracle_units, record_margin, rel_rms, sample_units

pytestmark = pytest.mark.gpu

DT = {"bf16": torch.bfloat16, "f32": torch.float32}


def _run_prefill(inp, C, S_out_alias=False):
    S0 = inp.get("S0")
    if S_out_alias and S0 is not None:
        return kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], S0,
                             inp.get("cu_seqlens"), C, S_out=S0)
    return kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], S0,
                         inp.get("cu_seqlens"), C)


# ---------------------------------------------------------------- prefill, small
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("T", [1, 7, 16, 17, 63, 64, 65, 130])
def test_prefill_small_shapes(cuda_device, dtype, d, T):
    inp = W.make_prefill(2, T, 3, d, d, dtype, -3.0, 1.0, 0.05, seed=100 + T + d, device=cuda_device)
    for C in (16, 32, 64):
        o, S = _run_prefill(inp, C)
        torch.cuda.synchronize()
        units = [(n, h) for n in range(2) for h in range(3)]
        compare_units(inp, o, S, units, TOL[DT[dtype]])


@pytest.mark.parametrize("dtype,d", [("f32", 32), ("bf16", 128), ("bf16", 64)])
def test_prefill_varlen_small(cuda_device, dtype, d):
    lens = (0, 1, 17, 64, 65, 100, 3)
    inp = W.make_prefill(1, sum(lens), 2, d, d, dtype, -3.0, 1.0, 0.05, seed=7, device=cuda_device,
                         lengths=lens)
    o, S = _run_prefill(inp, 64)
    torch.cuda.synchronize()
    units = [(n, h) for n in range(len(lens)) for h in range(2)]
    compare_units(inp, o, S, units, TOL[DT[dtype]])
    # the empty sequence hands its initial state through unchanged
    assert torch.equal(S[0], inp["S0"][0])


def test_prefill_oracle_small_config(cuda_device):
    """fp32, B1 H2 T256 d32, C=16: every unit, 1e-4."""
    w = W.ORACLE_SMALL
    inp = W.make_workload(w, cuda_device)
    for C in (16, 32, 64):
        o, S = _run_prefill(inp, C)
        torch.cuda.synchronize()
        compare_units(inp, o, S, [(0, 0), (0, 1)], 1e-4)


def test_prefill_state_aliasing_and_zero_length(cuda_device):
    inp = W.make_prefill(2, 40, 2, 64, 64, "bf16", -3.0, 1.0, 0.05, seed=3, device=cuda_device)
    o_ref, S_ref = _run_prefill(inp, 32)
    S0 = inp["S0"].clone()
    o2, S2 = _run_prefill(dict(inp, S0=S0), 32, S_out_alias=True)
    torch.cuda.synchronize()
    assert S2.data_ptr() == S0.data_ptr()
    assert torch.equal(S2, S_ref) and torch.equal(o2, o_ref)
    # T == 0: the state is handed through
    empty = W.make_prefill(2, 0, 2, 64, 64, "bf16", -3.0, 1.0, 0.05, seed=4, device=cuda_device)
    _, S = _run_prefill(empty, 64)
    torch.cuda.synchronize()
    assert torch.equal(S, empty["S0"])


def test_prefill_split_invariance(cuda_device):
    """prefill(T1) then prefill(T2) from its final state == prefill(T1 + T2)."""
    inp = W.make_prefill(1, 200, 4, 128, 128, "bf16", -4.0, 1.0, 0.02, seed=5, device=cuda_device)
    o, S = _run_prefill(inp, 64)
    cut = 77
    part = lambda x, a, b: x[:, a:b].contiguous()
    first = {n: part(inp[n], 0, cut) for n in ("q", "k", "v", "g", "beta")}
    second = {n: part(inp[n], cut, 200) for n in ("q", "k", "v", "g", "beta")}
    o1, S1 = _run_prefill(dict(first, S0=inp["S0"]), 64)
    o2, S2 = _run_prefill(dict(second, S0=S1), 64)
    torch.cuda.synchronize()
    assert rel_rms(torch.cat([o1, o2], 1).float().cpu(), o.float().cpu()) < 1e-2
    assert rel_rms(S2.cpu(), S.cpu()) < 1e-2
    compare_units(inp, o, S, [(0, h) for h in range(4)], 1e-2)


@pytest.mark.parametrize("g_rate", [1.2, 1.3])
def test_prefill_tc_chunk_decay_range_edges(cuda_device, g_rate):
    """Per-token log-decay close to -g_rate on every channel: a full 64-token
    chunk decays by about -76.8 (inside the single-reference range of the
    tensor-core path, factors up to e^76.8) or -83.2 (outside it: the chunk
    takes the 16-token block references).  T = 200 ends in an 8-token chunk
    that decays by ~-10, so the -83.2 case mixes both forms in one launch."""
    inp = W.make_prefill(2, 200, 4, 128, 128, "bf16", -3.0, 1.0, 0.05, seed=21, device=cuda_device)
    gen = torch.Generator(device=cuda_device).manual_seed(22)
    u = torch.rand(inp["g"].shape, generator=gen, device=cuda_device)
    inp["g"] = (-g_rate * (1.0 - 0.005 * u)).contiguous()
    o, S = _run_prefill(inp, 64)
    torch.cuda.synchronize()
    assert torch.isfinite(o).all() and torch.isfinite(S).all()
    compare_units(inp, o, S, [(n, h) for n in range(2) for h in range(4)], 1e-2)


def test_prefill_tc_steep_random_decay(cuda_device):
    """Random steep gates (log-decay about -2 per token, up to -2.7): every
    full chunk of the tensor-core path takes the block-reference form."""
    inp = W.make_prefill(2, 300, 4, 128, 128, "bf16", 1.8, 0.2, 0.05, seed=23, device=cuda_device)
    assert float(inp["g"].min()) > -5.0
    o, S = _run_prefill(inp, 64)
    torch.cuda.synchronize()
    assert torch.isfinite(o).all() and torch.isfinite(S).all()
    compare_units(inp, o, S, [(n, h) for n in range(2) for h in range(4)], 1e-2)


# ------------------------------------------------------------ prefill, full size
def test_prefill_h16_full(cuda_device):
    """bf16 B1 H16 T4096 d128, random initial state: all 16 units."""
    w = W.PREFILL_H16
    inp = W.make_workload(w, cuda_device)
    o, S = _run_prefill(inp, w.chunk)
    torch.cuda.synchronize()
    compare_units(inp, o, S, [(0, h) for h in range(w.H)], 1e-2)


def test_prefill_b8_sampled(cuda_device):
    """bf16 B8 H32 T8192 d128 (the benchmark workload, same launch): 40 seeded
    units, the first and the last always included."""
    w = W.PREFILL_B8
    inp = W.make_workload(w, cuda_device)
    o, S = _run_prefill(inp, w.chunk)
    torch.cuda.synchronize()
    units = sample_units(w.B, w.H, 40, seed=11, must=[(0, 0), (w.B - 1, w.H - 1)])
    compare_units(inp, o, S, units, 1e-2)
    assert torch.isfinite(o).all() and torch.isfinite(S).all()


def test_prefill_varlen_sampled(cuda_device):
    """16 packed sequences (~512K tokens), H32: the longest and the shortest
    sequence on four heads each, plus seeded units (40 in all)."""
    w = W.PREFILL_VARLEN
    inp = W.make_workload(w, cuda_device)
    o, S = _run_prefill(inp, w.chunk)
    torch.cuda.synchronize()
    lens = list(w.lengths)
    longest, shortest = int(np.argmax(lens)), int(np.argmin(lens))
    must = [(longest, h) for h in (0, 3, 17, 31)] + [(shortest, h) for h in (0, 9, 17, 30)]
    units = sample_units(w.num_seqs, w.H, 40, seed=12, must=must)
    compare_units(inp, o, S, units, 1e-2)
    assert torch.isfinite(o).all() and torch.isfinite(S).all()


# ------------------------------------------------------------------------ decode
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [32, 64, 128])
def test_decode_small(cuda_device, dtype, d):
    N, H, steps = 3, 2, 40
    S = W.make_decode_state(N, H, d, d, 0.05, seed=20 + d, device=cuda_device)
    S0 = S.clone()
    x = W.make_decode_steps(N, H, d, d, steps, dtype, seed=21 + d, device=cuda_device)
    outs = []
    for t in range(steps):
        outs.append(kda.recurrent_step(x["q"][t], x["k"][t], x["v"][t], x["g"][t], x["beta"][t], S))
    torch.cuda.synchronize()
    o = torch.stack(outs, 1)  # [N, steps, H, dv]
    # the oracle sees the steps as one prefill per sequence
    as_prefill = {n: x[n].transpose(0, 1).contiguous() for n in ("q", "k", "v", "g", "beta")}
    ro, rS = oracle.recurrent(as_prefill["q"], as_prefill["k"], as_prefill["v"], as_prefill["g"],
                              as_prefill["beta"], S0)
    tol = TOL[DT[dtype]]
    assert oracle.rel_rms_per_slice(o.float().cpu().numpy(), ro) <= tol
    assert oracle.rel_rms_per_slice(S.cpu().numpy(), rS) <= tol


def test_decode_full_all_units(cuda_device):
    """256 sequences x 32 heads, d128, 1024 in-place steps (the benchmark's
    decode launch, same inputs): every one of the 8,192 units, o at steps 1,
    2, 8, 64 and 1024 and the final state, against the oracle run on the same
    steps as one prefill per unit (in batches of units, to bound host memory)."""
    w = W.DECODE
    N, H, d, steps = w.B, w.H, w.dk, w.T
    S = W.make_decode_state(N, H, d, d, w.s0_std, seed=w.seed, device=cuda_device)
    S0 = S.clone()
    xs = W.make_decode_steps(N, H, d, d, steps, w.dtype, w.g_mu, w.g_sigma, seed=w.seed, device=cuda_device)
    keep_steps = (0, 1, 7, 63, steps - 1)
    o_kept = {}
    for t in range(steps):
        o = kda.recurrent_step(xs["q"][t], xs["k"][t], xs["v"][t], xs["g"][t], xs["beta"][t], S)
        if t in keep_steps:
            o_kept[t] = o.float().cpu()
    torch.cuda.synchronize()
    S_gpu = S.cpu()
    worst_o = worst_S = 0.0
    batch = 256
    flat = lambda x: x.reshape(steps, N * H, *x.shape[3:])  # [steps, units, ...]
    for u0 in range(0, N * H, batch):
        sel = slice(u0, u0 + batch)
        seq = {n: flat(xs[n])[:, sel].transpose(0, 1).unsqueeze(2).cpu() for n in ("q", "k", "v", "g", "beta")}
        S0_b = S0.reshape(N * H, d, d)[sel].unsqueeze(1).cpu()
        ro, rS = oracle.recurrent(seq["q"], seq["k"], seq["v"], seq["g"], seq["beta"], S0_b)
        for t in keep_steps:
            og = o_kept[t].reshape(N * H, d)[sel].numpy()
            worst_o = max(worst_o, oracle.rel_rms_per_slice(og[:, None, None, :], ro[:, t:t + 1]))
        worst_S = max(worst_S, oracle.rel_rms_per_slice(S_gpu.reshape(N * H, d, d)[sel].unsqueeze(1).numpy(), rS))
    record_margin(worst_o, worst_S, 1e-2, N * H)
    assert worst_o <= 1e-2 and worst_S <= 1e-2, (worst_o, worst_S)


def test_decode_equals_prefill(cuda_device):
    N, H, d, T = 2, 4, 128, 50
    inp = W.make_prefill(N, T, H, d, d, "bf16", -3.0, 1.0, 0.05, seed=30, device=cuda_device)
    o_p, S_p = _run_prefill(inp, 64)
    S = inp["S0"].clone()
    outs = []
    for t in range(T):
        outs.append(kda.recurrent_step(inp["q"][:, t].contiguous(), inp["k"][:, t].contiguous(),
                                       inp["v"][:, t].contiguous(), inp["g"][:, t].contiguous(),
                                       inp["beta"][:, t].contiguous(), S))
    torch.cuda.synchronize()
    o_d = torch.stack(outs, 1)
    assert rel_rms(o_d.float().cpu(), o_p.float().cpu()) < 1e-2
    assert rel_rms(S.cpu(), S_p.cpu()) < 1e-2
    assert kda.device_error() == 0
