"""GPU parity on the method's degenerate cases, for the tensor-core path (bf16,
d128, C64) and the fp32 path: beta = 0 (no writes: the state only decays),
g = 0 (no decay), zero key / query rows, a single token, and beta = 1 with
repeated keys (each write fully replaces the value stored along that key)."""
import pytest
import torch

import kimi_delta_attention_31_b200 as kda
import kda_workloads as W
from parity_util import TOL, compare_units

pytestmark = pytest.mark.gpu

PATHS = [("bf16", 128, 64), ("f32", 32, 16)]


def _run(inp, C):
    return kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp.get("S0"), None, C)


@pytest.mark.parametrize("dtype,d,C", PATHS)
def test_beta_zero_only_decays_the_state(cuda_device, dtype, d, C):
    inp = W.make_prefill(2, 130, 2, d, d, dtype, -3.0, 1.0, 0.1, seed=700, device=cuda_device)
    inp["beta"].zero_()
    o, S = _run(inp, C)
    torch.cuda.synchronize()
    compare_units(inp, o, S, [(n, h) for n in range(2) for h in range(2)], TOL[inp["q"].dtype])
    # S_T = Diag(exp(sum_t g_t)) S0 exactly in this case
    decay = torch.exp(inp["g"].double().sum(1))                     # [B, H, dk]
    ref = decay.unsqueeze(-1) * inp["S0"].double()
    err = (S.double() - ref).norm() / ref.norm()
    assert err < TOL[inp["q"].dtype]


@pytest.mark.parametrize("dtype,d,C", PATHS)
def test_no_decay(cuda_device, dtype, d, C):
    inp = W.make_prefill(1, 150, 2, d, d, dtype, -3.0, 1.0, 0.05, seed=701, device=cuda_device)
    inp["g"].zero_()
    o, S = _run(inp, C)
    torch.cuda.synchronize()
    compare_units(inp, o, S, [(0, 0), (0, 1)], TOL[inp["q"].dtype])


@pytest.mark.parametrize("dtype,d,C", PATHS)
def test_zero_key_and_query_rows(cuda_device, dtype, d, C):
    inp = W.make_prefill(1, 100, 2, d, d, dtype, -3.0, 1.0, 0.05, seed=702, device=cuda_device)
    inp["k"][0, 10:40] = 0
    inp["q"][0, 30:70] = 0
    o, S = _run(inp, C)
    torch.cuda.synchronize()
    assert torch.count_nonzero(o[0, 30:70]) == 0  # o_t = S_t^T q_t = 0 for q_t = 0
    compare_units(inp, o, S, [(0, 0), (0, 1)], TOL[inp["q"].dtype])


@pytest.mark.parametrize("dtype,d,C", PATHS)
def test_single_token(cuda_device, dtype, d, C):
    inp = W.make_prefill(3, 1, 2, d, d, dtype, -3.0, 1.0, 0.05, seed=703, device=cuda_device)
    o, S = _run(inp, C)
    torch.cuda.synchronize()
    compare_units(inp, o, S, [(n, h) for n in range(3) for h in range(2)], TOL[inp["q"].dtype])


@pytest.mark.parametrize("dtype,d,C", PATHS)
def test_full_replacement_with_repeated_keys(cuda_device, dtype, d, C):
    """beta = 1, no decay, the same unit key every token: the state's value
    along k is replaced each step, so S_t^T k = v_t and o_t = S_t^T q."""
    inp = W.make_prefill(1, 90, 1, d, d, dtype, -3.0, 1.0, 0.0, seed=704, device=cuda_device)
    inp["k"][:] = inp["k"][:, :1]
    inp["beta"].fill_(1.0)
    inp["g"].zero_()
    o, S = _run(inp, C)
    torch.cuda.synchronize()
    # With one key every entry below the diagonal of A is |k|^2, so every
    # subdiagonal entry of T diag(beta) is the same -|k|^2 and the outputs are
    # telescoping sums over up to 64 rows: a rounding of T diag(beta) or of the
    # corrected errors to bf16 would add up coherently.  The tensor-core prefill
    # feeds both to its MMAs as bf16 hi + lo pairs, so the bf16 tolerance holds.
    compare_units(inp, o, S, [(0, 0)], TOL[inp["q"].dtype])
    kk = inp["k"][0, 0, 0].float()
    readback = S[0, 0].T @ kk * (1.0 / (kk @ kk))  # S^T k / |k|^2 with |k| ~ 1 after rounding
    ref = inp["v"][0, -1, 0].float()
    assert (readback - ref).norm() / ref.norm() < 2e-2
