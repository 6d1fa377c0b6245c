"""Sequence parallelism of the tensor-core prefill: each sequence split into
segments whose affine state maps are formed in parallel and chained from S0.
Parity against the fp64 oracle, and against the unsplit GPU run."""
import pytest
import torch

import kimi_delta_attention_31_b200 as kda
import kda_workloads as W
from parity_util import compare_units, rel_rms, sample_units

pytestmark = pytest.mark.gpu


@pytest.fixture
def segments():
    yield kda.set_segment_chunks
    kda.set_segment_chunks(0)


def _run(inp):
    return kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp.get("S0"), None, 64)


@pytest.mark.parametrize("L", [1, 8, 16, 46])
def test_forced_segments_match_oracle_and_unsplit(cuda_device, segments, L):
    """B2 H3 T3000 (47 chunks, ragged last chunk), random S0."""
    inp = W.make_prefill(2, 3000, 3, 128, 128, "bf16", -4.0, 1.0, 0.05, seed=80 + L, device=cuda_device)
    segments(-1)
    o_ref, S_ref = _run(inp)
    segments(L)
    assert kda.segment_chunks(2, 3000, 3) == L
    o, S = _run(inp)
    torch.cuda.synchronize()
    compare_units(inp, o, S, [(n, h) for n in range(2) for h in range(3)], 1e-2)
    assert rel_rms(o.float().cpu(), o_ref.float().cpu()) < 1e-2
    assert rel_rms(S.cpu(), S_ref.cpu()) < 1e-2


def test_segments_with_zero_state_and_gdn(cuda_device, segments):
    inp = W.make_prefill(1, 1500, 2, 128, 128, "bf16", -4.0, 1.0, 0.0, seed=81, device=cuda_device,
                         scalar_gate=True)
    segments(5)
    o, S = kda.gdn_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], None, None, 64)
    torch.cuda.synchronize()
    compare_units(inp, o, S, [(0, 0), (0, 1)], 1e-2)


def test_automatic_segments_on_a_long_sequence(cuda_device, segments):
    """B1 H4 T65536: four units cannot fill the GPU, so the prefill splits
    each sequence by itself; sampled heads against the oracle."""
    segments(0)
    L = kda.segment_chunks(1, 65536, 4)
    assert L > 0
    inp = W.make_prefill(1, 65536, 4, 128, 128, "bf16", -5.0, 1.5, 0.02, seed=82, device=cuda_device)
    o, S = _run(inp)
    torch.cuda.synchronize()
    compare_units(inp, o, S, [(0, 0), (0, 3)], 1e-2)
    assert torch.isfinite(o).all() and torch.isfinite(S).all()
    assert kda.device_error() == 0


def test_no_segments_where_units_fill_the_gpu(cuda_device, segments):
    segments(0)
    assert kda.segment_chunks(8, 8192, 32) == 0      # the headline shape
    assert kda.segment_chunks(1, 520998, 32, 16) == 0  # packed inputs are never split
    assert kda.segment_chunks(1, 2048, 4) == 0        # 32 chunks: too short to pay off
    assert kda.segment_chunks(1, 4096, 16) == 16      # 64 chunks, 16 units: measured 0.247 -> 0.185 ms
    assert kda.segment_chunks(4, 4096, 16) == 0       # 64 units: measured no gain


def test_segments_with_the_final_state_aliasing_the_initial_state(cuda_device, segments):
    """S_out may alias S0: with segments, the last segment writes S_out while
    other segments still run, so no segment may read S0 itself then."""
    inp = W.make_prefill(2, 2000, 3, 128, 128, "bf16", -4.0, 1.0, 0.05, seed=83, device=cuda_device)
    segments(4)
    o_ref, S_ref = _run(inp)
    S0 = inp["S0"].clone()
    o2, S2 = kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], S0, None, 64, S_out=S0)
    torch.cuda.synchronize()
    assert S2.data_ptr() == S0.data_ptr()
    assert torch.equal(o2, o_ref) and torch.equal(S2, S_ref)
