"""Device-side checks of cu_seqlens.  The packed layout's table lives on the
device, so the host cannot check it without a synchronisation; the kernels
check it instead.  Every malformed table here keeps its values inside the
buffers the call was given, so that even a missed check could not read or
write out of bounds: the test looks only for the reported error and for the
outputs being left alone."""
import pytest
import torch

import kimi_delta_attention_31_b200 as kda
import kda_workloads as W
from parity_util import TOL, compare_units

pytestmark = pytest.mark.gpu

LENS = (100, 40, 160)  # 300 tokens
BAD_TABLES = {
    "non_monotone": [0, 100, 50, 300],
    "short_total": [0, 100, 140, 200],
    "nonzero_start": [10, 100, 140, 300],
}


def _packed(device, dtype="bf16", d=128):
    return W.make_prefill(1, sum(LENS), 2, d, d, dtype, -3.0, 1.0, 0.05, seed=61, device=device, lengths=LENS)


@pytest.mark.parametrize("local_kernel", [0, 1])
@pytest.mark.parametrize("name", sorted(BAD_TABLES))
def test_tensor_core_path_rejects_malformed_table(cuda_device, name, local_kernel):
    x = _packed(cuda_device)
    assert kda.device_error() == 0
    kda.set_local_kernel(local_kernel)
    try:
        bad = torch.tensor(BAD_TABLES[name], dtype=torch.int32, device=cuda_device)
        o = torch.full_like(x["v"], 7.0)
        S_out = torch.full_like(x["S0"], 3.0)
        kda.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], bad, 64, o=o, S_out=S_out)
        assert kda.device_error() == 1  # KDA_ERR_INVALID_ARG, read and cleared
        assert bool((o == 7.0).all()) and bool((S_out == 3.0).all())
        # the context stays usable: the same call with the valid table matches the oracle
        o2, S2 = kda.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], x["cu_seqlens"], 64)
        torch.cuda.synchronize()
        assert kda.device_error() == 0
        compare_units(x, o2, S2, [(n, h) for n in range(len(LENS)) for h in range(2)], TOL[torch.bfloat16])
    finally:
        kda.set_local_kernel(0)


def test_fp32_path_treats_out_of_range_sequence_as_empty(cuda_device):
    x = _packed(cuda_device, "f32", 32)
    bad = torch.tensor(BAD_TABLES["non_monotone"], dtype=torch.int32, device=cuda_device)
    o = torch.full_like(x["v"], 7.0)
    _, S = kda.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], bad, 16, o=o)
    assert kda.device_error() == 1
    # sequence 1 ([100, 50)) is empty: its final state is its initial state
    assert torch.equal(S[1], x["S0"][1])
    assert torch.isfinite(o).all()
