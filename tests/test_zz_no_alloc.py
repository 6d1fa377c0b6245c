"""kda_chunk_fwd_noalloc: the prefill for callers that cannot allocate device
memory (for example a plug-in handed only input and output pointers by a host
framework that owns the device memory pool).  It must give the same results
as kda_chunk_fwd with a caller-allocated workspace, call after call (its
built-in scratch array is reused), and refuse sizes its array cannot hold.

This file is named so that pytest collects it last."""
import pytest
import torch

import kimi_delta_attention_31_b200 as kda
import kda_workloads as W
from parity_util import rel_rms

pytestmark = pytest.mark.gpu

TOL = 1e-2  # the bf16 tolerance of the parity tests


def _inputs(seed, device):
    # tensor-core shape (bf16, d=128, C=64), ragged last chunk, random initial state:
    # 2 x 11 chunks x 8 heads = 176 (chunk, head) images, well inside the built-in array
    return W.make_prefill(2, 700, 8, 128, 128, "bf16", -4.0, 1.0, 0.02, seed=seed, device=device)


def test_noalloc_matches_workspace_entry_point_twice(cuda_device):
    for call, seed in enumerate((901, 902)):
        x = _inputs(seed, cuda_device)
        ref_o, ref_S = kda.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], None, 64)
        o, S = kda.chunk_fwd_noalloc(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], None, 64)
        torch.cuda.synchronize()
        assert torch.isfinite(o.float()).all() and torch.isfinite(S).all()
        eo = rel_rms(o.float().cpu().numpy(), ref_o.float().cpu().numpy())
        eS = rel_rms(S.cpu().numpy(), ref_S.cpu().numpy())
        assert eo <= TOL and eS <= TOL, f"call {call}: o {eo:.3e}, S {eS:.3e}"


def test_noalloc_packed_sequences(cuda_device):
    lens = (64, 1, 130, 0, 77)
    x = W.make_prefill(1, sum(lens), 4, 128, 128, "bf16", -4.0, 1.0, 0.02, seed=903, device=cuda_device,
                       lengths=lens)
    ref_o, ref_S = kda.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], x["cu_seqlens"], 64)
    o, S = kda.chunk_fwd_noalloc(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], x["cu_seqlens"], 64)
    torch.cuda.synchronize()
    assert rel_rms(o.float().cpu().numpy(), ref_o.float().cpu().numpy()) <= TOL
    assert rel_rms(S.cpu().numpy(), ref_S.cpu().numpy()) <= TOL


def test_noalloc_rejects_sizes_beyond_its_array(cuda_device):
    need = kda.workspace_size(1, 8192, 16, 128, 128, 0, 64, torch.bfloat16)
    assert need > kda.NOALLOC_SCRATCH_BYTES
    x = W.make_prefill(1, 8192, 16, 128, 128, "bf16", seed=904, device=cuda_device)
    with pytest.raises(kda.KDAError) as err:
        kda.chunk_fwd_noalloc(x["q"], x["k"], x["v"], x["g"], x["beta"])
    assert err.value.status == 4 and "built-in" in str(err.value)
