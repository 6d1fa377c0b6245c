"""GPU parity of the Gated DeltaNet entry points (one gate per token and
head): kda_gdn_chunk_fwd and kda_gdn_recurrent_step against the fp64 oracle
(the recurrence with the gate broadcast over key channels), plus the identity
with the per-channel entry points fed the broadcast gate."""
import pytest
import torch

import kimi_delta_attention_31_b200 as kda
import kda_workloads as W
import oracle
from parity_util import TOL, compare_units, rel_rms, sample_units

pytestmark = pytest.mark.gpu

DT = {"bf16": torch.bfloat16, "f32": torch.float32}


def _gdn(inp, C):
    return kda.gdn_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp.get("S0"),
                             inp.get("cu_seqlens"), C)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("T", [1, 17, 64, 130])
def test_gdn_prefill_small_shapes(cuda_device, dtype, d, T):
    inp = W.make_prefill(2, T, 3, d, d, dtype, -3.0, 1.0, 0.05, seed=300 + T + d, device=cuda_device,
                         scalar_gate=True)
    assert inp["g"].shape == (2, T, 3)
    for C in (16, 32, 64):
        o, S = _gdn(inp, C)
        torch.cuda.synchronize()
        compare_units(inp, o, S, [(n, h) for n in range(2) for h in range(3)], TOL[DT[dtype]])


@pytest.mark.parametrize("dtype,d", [("f32", 32), ("bf16", 128)])
def test_gdn_prefill_varlen_small(cuda_device, dtype, d):
    lens = (0, 1, 17, 64, 65, 100, 3)
    inp = W.make_prefill(1, sum(lens), 2, d, d, dtype, -3.0, 1.0, 0.05, seed=31, device=cuda_device,
                         lengths=lens, scalar_gate=True)
    o, S = _gdn(inp, 64)
    torch.cuda.synchronize()
    compare_units(inp, o, S, [(n, h) for n in range(len(lens)) for h in range(2)], TOL[DT[dtype]])
    assert torch.equal(S[0], inp["S0"][0])


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("bf16", 64), ("f32", 32)])
def test_gdn_equals_kda_with_broadcast_gate(cuda_device, dtype, d):
    """The scalar-gate entry point reads g[t, h] where the per-channel one reads
    g[t, h, c]; fed the broadcast gate, the same kernel gives the same bits --
    for each of the two chunk-local kernels of the tensor-core path (the
    warp-specialised default and the two-CTA one), which agree with each
    other to rounding (they sum G in different orders)."""
    inp = W.make_prefill(2, 150, 4, d, d, dtype, -3.0, 1.0, 0.05, seed=32, device=cuda_device,
                         scalar_gate=True)
    g_full = inp["g"].unsqueeze(-1).expand(2, 150, 4, d).contiguous()
    res = []
    for variant in (0, 1):
        kda.set_local_kernel(variant)
        try:
            o1, S1 = _gdn(inp, 64)
            o2, S2 = kda.chunk_fwd(inp["q"], inp["k"], inp["v"], g_full, inp["beta"], inp["S0"], None, 64)
        finally:
            kda.set_local_kernel(0)
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(S1, S2)
        res.append((o1, S1))
    (oa, Sa), (ob, Sb) = res
    assert rel_rms(oa.float().cpu(), ob.float().cpu()) < 1e-3 and rel_rms(Sa.cpu(), Sb.cpu()) < 1e-3


def test_gdn_prefill_b8_sampled(cuda_device):
    """bf16 B8 H32 T8192 d128 with one gate per token and head (the benchmark's
    Gated DeltaNet launch): 8 sampled units."""
    w = W.GDN_PREFILL_B8
    inp = W.make_workload(w, cuda_device)
    o, S = _gdn(inp, w.chunk)
    torch.cuda.synchronize()
    units = sample_units(w.B, w.H, 8, seed=14, must=[(0, 0), (w.B - 1, w.H - 1)])
    compare_units(inp, o, S, units, 1e-2)
    assert torch.isfinite(o).all() and torch.isfinite(S).all()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [32, 128])
def test_gdn_decode_small(cuda_device, dtype, d):
    N, H, steps = 3, 2, 40
    S = W.make_decode_state(N, H, d, d, 0.05, seed=40 + d, device=cuda_device)
    S0 = S.clone()
    x = W.make_decode_steps(N, H, d, d, steps, dtype, seed=41 + d, device=cuda_device, scalar_gate=True)
    assert x["g"].shape == (steps, N, H)
    outs = [kda.gdn_recurrent_step(x["q"][t], x["k"][t], x["v"][t], x["g"][t], x["beta"][t], S)
            for t in range(steps)]
    torch.cuda.synchronize()
    o = torch.stack(outs, 1)
    as_prefill = {n: x[n].transpose(0, 1).contiguous() for n in ("q", "k", "v", "g", "beta")}
    ro, rS = oracle.gdn_recurrent(as_prefill["q"], as_prefill["k"], as_prefill["v"], as_prefill["g"],
                                  as_prefill["beta"], S0)
    tol = TOL[DT[dtype]]
    assert oracle.rel_rms_per_slice(o.float().cpu().numpy(), ro) <= tol
    assert oracle.rel_rms_per_slice(S.cpu().numpy(), rS) <= tol


def test_gdn_decode_equals_prefill(cuda_device):
    N, H, d, T = 2, 4, 128, 50
    inp = W.make_prefill(N, T, H, d, d, "bf16", -3.0, 1.0, 0.05, seed=33, device=cuda_device,
                         scalar_gate=True)
    o_p, S_p = _gdn(inp, 64)
    S = inp["S0"].clone()
    outs = [kda.gdn_recurrent_step(inp["q"][:, t].contiguous(), inp["k"][:, t].contiguous(),
                                   inp["v"][:, t].contiguous(), inp["g"][:, t].contiguous(),
                                   inp["beta"][:, t].contiguous(), S) for t in range(T)]
    torch.cuda.synchronize()
    assert rel_rms(torch.stack(outs, 1).float().cpu(), o_p.float().cpu()) < 1e-2
    assert rel_rms(S.cpu(), S_p.cpu()) < 1e-2
