"""GPU parity of the fused-preparation entry points (kda_chunk_fwd_prep,
kda_recurrent_step_prep): raw q, k (unnormalised), raw gate logits a (fp32 or
bf16) and raw beta logits b go in; the fp64 oracle prepares the same raw
values (L2 normalisation, log alpha = -softplus(a), beta = sigmoid(b)) and
runs the recurrence."""
import pytest
import torch

import kimi_delta_attention_31_b200 as kda
import kda_workloads as W
import oracle
from parity_util import TOL, compare_units_prep, sample_units

pytestmark = pytest.mark.gpu

DT = {"bf16": torch.bfloat16, "f32": torch.float32}


def _prep(inp, C):
    return kda.chunk_fwd_prep(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"], inp.get("S0"),
                              inp.get("cu_seqlens"), C)


@pytest.mark.parametrize("a_dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("bf16", 64), ("f32", 32), ("f32", 128)])
@pytest.mark.parametrize("T", [1, 17, 65, 130])
def test_prep_prefill_small_shapes(cuda_device, a_dtype, dtype, d, T):
    inp = W.make_prefill_raw(2, T, 3, d, d, dtype, -3.0, 1.0, a_dtype, 0.05, seed=500 + T + d,
                             device=cuda_device)
    for C in ((16, 64) if dtype == "f32" else (64,)):
        o, S = _prep(inp, C)
        torch.cuda.synchronize()
        compare_units_prep(inp, o, S, [(n, h) for n in range(2) for h in range(3)], TOL[DT[dtype]])


def test_prep_prefill_varlen_small(cuda_device):
    lens = (0, 1, 17, 64, 65, 100, 3)
    inp = W.make_prefill_raw(1, sum(lens), 2, 128, 128, "bf16", -3.0, 1.0, "bf16", 0.05, seed=51,
                             device=cuda_device, lengths=lens)
    o, S = _prep(inp, 64)
    torch.cuda.synchronize()
    compare_units_prep(inp, o, S, [(n, h) for n in range(len(lens)) for h in range(2)], 1e-2)
    assert torch.equal(S[0], inp["S0"][0])


def test_prep_handles_zero_rows_and_extreme_logits(cuda_device):
    """A zero q or k row stays zero after normalisation; gate logits of 15
    (log alpha ~ -15 for 4 tokens: ~-60 over their 16-token block, inside the
    tensor-core path's domain) and -40 (alpha ~ 1), and beta logits of +-30
    stay finite and match."""
    inp = W.make_prefill_raw(1, 96, 2, 128, 128, "bf16", -3.0, 1.0, "f32", 0.05, seed=52, device=cuda_device)
    inp["q"][0, 5, 0] = 0
    inp["k"][0, 9, 1] = 0
    inp["a"][0, 20:24] = 15.0
    inp["a"][0, 30:34] = -40.0
    inp["b"][0, 40, 0] = 30.0
    inp["b"][0, 41, 1] = -30.0
    o, S = _prep(inp, 64)
    torch.cuda.synchronize()
    assert torch.isfinite(o).all() and torch.isfinite(S).all()
    compare_units_prep(inp, o, S, [(0, 0), (0, 1)], 1e-2)


def test_prep_prefill_b8_sampled(cuda_device):
    """The benchmark's fused-preparation launch (B8 H32 T8192 d128, bf16 gate
    logits): 8 sampled units."""
    w = W.PREP_PREFILL_B8
    inp = W.make_workload(w, cuda_device)
    o, S = _prep(inp, w.chunk)
    torch.cuda.synchronize()
    units = sample_units(w.B, w.H, 8, seed=15, must=[(0, 0), (w.B - 1, w.H - 1)])
    compare_units_prep(inp, o, S, units, 1e-2)
    assert torch.isfinite(o).all() and torch.isfinite(S).all()


@pytest.mark.parametrize("a_dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 32)])
def test_prep_decode_small(cuda_device, a_dtype, dtype, d):
    N, H, steps = 3, 2, 30
    raw = W.make_prefill_raw(N, steps, H, d, d, dtype, -3.0, 1.0, a_dtype, 0.05, seed=53 + d,
                             device=cuda_device)
    S = raw["S0"].clone()
    outs = [kda.recurrent_step_prep(raw["q"][:, t].contiguous(), raw["k"][:, t].contiguous(),
                                    raw["v"][:, t].contiguous(), raw["a"][:, t].contiguous(),
                                    raw["b"][:, t].contiguous(), S) for t in range(steps)]
    torch.cuda.synchronize()
    o = torch.stack(outs, 1)
    ro, rS = oracle.recurrent_prep(raw["q"], raw["k"], raw["v"], raw["a"], raw["b"], raw["S0"])
    tol = TOL[DT[dtype]]
    assert oracle.rel_rms_per_slice(o.float().cpu().numpy(), ro) <= tol
    assert oracle.rel_rms_per_slice(S.cpu().numpy(), rS) <= tol
