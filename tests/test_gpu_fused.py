"""GPU parity of the single-pass tensor-core prefill (kda_set_prefill_path(1)):
one persistent kernel per call that builds every chunk's operands, solves
(I + A) and carries the state through the chunks of each (sequence, head) unit
in tensor memory.  Against the fp64 oracle at the bf16 tolerance, and against
the two-kernel path on the same inputs, across shapes with ragged chunks,
packed sequences (empty ones included), chunks past the single-reference decay
range, the per-token gate, raw projections, S_out aliasing S0, and more units
than SMs (the dynamic unit schedule); and in its role as the two-kernel
path's precise fallback for chunks with near-parallel keys."""
import numpy as np
import pytest
import torch

import kimi_delta_attention_31_b200 as kda
import kda_workloads as W
from parity_util import compare_units, compare_units_prep, rel_rms

pytestmark = pytest.mark.gpu


def _on_path(path, fn):
    kda.set_prefill_path(path)
    try:
        out = fn()
    finally:
        kda.set_prefill_path(kda.PATH_AUTO)
    torch.cuda.synchronize()
    assert kda.device_error() == 0
    return out


def _both_paths(fn):
    return _on_path(kda.PATH_FUSED, fn), _on_path(kda.PATH_TWO_KERNEL, fn)


def _prefill(inp, cu=None, **kw):
    return lambda: kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp.get("S0"), cu, 64, **kw)


@pytest.mark.parametrize("B,T,H,s0", [(1, 1, 1, 0.05), (1, 64, 2, 0.0), (2, 65, 3, 0.05), (2, 200, 4, 0.05),
                                      (3, 130, 3, 0.0), (2, 1000, 5, 0.02), (1, 4096, 2, 0.02)])
def test_fused_matches_oracle_and_two_kernel_path(cuda_device, B, T, H, s0):
    inp = W.make_prefill(B, T, H, 128, 128, "bf16", -4.0, 1.0, s0, seed=500 + T + H, device=cuda_device)
    (o1, S1), (o2, S2) = _both_paths(_prefill(inp))
    units = [(n, h) for n in range(B) for h in range(H)]
    compare_units(inp, o1, S1, units, 1e-2)
    assert rel_rms(o1.float().cpu(), o2.float().cpu()) < 1e-2
    assert rel_rms(S1.cpu(), S2.cpu()) < 1e-2


def test_fused_many_units_dynamic_schedule(cuda_device):
    """B4 H80 T300: 320 units on at most 148 CTAs, taken from the counter."""
    inp = W.make_prefill(4, 300, 80, 128, 128, "bf16", -4.0, 1.0, 0.02, seed=510, device=cuda_device)
    (o1, S1), (o2, S2) = _both_paths(_prefill(inp))
    compare_units(inp, o1, S1, [(0, 0), (1, 17), (2, 40), (3, 79), (3, 5), (0, 63)], 1e-2)
    assert rel_rms(o1.float().cpu(), o2.float().cpu()) < 1e-2
    assert rel_rms(S1.cpu(), S2.cpu()) < 1e-2


@pytest.mark.parametrize("frac", [0.1, 0.5, 1.0])
def test_fused_steep_chunks(cuda_device, frac):
    """Chunks whose decay on some channel is past -80 over the chunk take four
    block-reference MMAs and the Kbar form of the state update."""
    B, T, H = 2, 700, 4
    inp = W.make_prefill(B, T, H, 128, 128, "bf16", -4.0, 1.0, 0.05, seed=520, device=cuda_device)
    gen = torch.Generator(device=cuda_device).manual_seed(521 + int(10 * frac))
    nc = (T + 63) // 64
    steep = torch.rand((B, nc, H), generator=gen, device=cuda_device) < frac
    rate = torch.where(steep, torch.full_like(steep, 1.5, dtype=torch.float32),
                       torch.full_like(steep, 0.05, dtype=torch.float32)).repeat_interleave(64, dim=1)[:, :T]
    u = torch.rand(inp["g"].shape, generator=gen, device=cuda_device)
    inp["g"] = (-rate.unsqueeze(-1) * (1.0 - 0.005 * u)).contiguous()
    (o1, S1), (o2, S2) = _both_paths(_prefill(inp))
    assert torch.isfinite(o1.float()).all() and torch.isfinite(S1).all()
    compare_units(inp, o1, S1, [(n, h) for n in range(B) for h in range(H)], 1e-2)
    assert rel_rms(o1.float().cpu(), o2.float().cpu()) < 1e-2


@pytest.mark.parametrize("lens", [(0, 1, 17, 64, 65, 100, 3), (130,) * 40 + (0, 7), (4096, 1, 2000, 64)])
def test_fused_packed_sequences(cuda_device, lens):
    inp = W.make_prefill(1, sum(lens), 3, 128, 128, "bf16", -4.0, 1.0, 0.05, seed=530 + len(lens),
                         device=cuda_device, lengths=lens)
    (o1, S1), (o2, S2) = _both_paths(_prefill(inp, inp["cu_seqlens"]))
    units = [(n, h) for n in range(len(lens)) for h in range(3)]
    compare_units(inp, o1, S1, units[:30] + units[-6:], 1e-2)
    assert rel_rms(o1.float().cpu(), o2.float().cpu()) < 1e-2
    for n, L in enumerate(lens):  # an empty sequence hands its state through
        if L == 0:
            assert torch.equal(S1[n], inp["S0"][n])


def test_fused_gated_deltanet(cuda_device):
    inp = W.make_prefill(2, 300, 4, 128, 128, "bf16", -3.0, 1.0, 0.05, seed=540, device=cuda_device,
                         scalar_gate=True)
    fn = lambda: kda.gdn_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["S0"], None, 64)
    (o1, S1), (o2, S2) = _both_paths(fn)
    compare_units(inp, o1, S1, [(n, h) for n in range(2) for h in range(4)], 1e-2)
    assert rel_rms(o1.float().cpu(), o2.float().cpu()) < 1e-2


@pytest.mark.parametrize("a_dtype", ["f32", "bf16"])
def test_fused_prep(cuda_device, a_dtype):
    inp = W.make_prefill_raw(2, 333, 3, 128, 128, "bf16", -3.0, 1.0, a_dtype, 0.05, seed=550, device=cuda_device)
    fn = lambda: kda.chunk_fwd_prep(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"], inp["S0"], None, 64)
    (o1, S1), (o2, S2) = _both_paths(fn)
    compare_units_prep(inp, o1, S1, [(n, h) for n in range(2) for h in range(3)], 1e-2)
    assert rel_rms(o1.float().cpu(), o2.float().cpu()) < 1e-2


def test_fused_state_aliasing(cuda_device):
    inp = W.make_prefill(2, 150, 4, 128, 128, "bf16", -4.0, 1.0, 0.05, seed=560, device=cuda_device)
    o_ref, S_ref = _on_path(kda.PATH_FUSED, _prefill(inp))
    S0 = inp["S0"].clone()
    o2, S2 = _on_path(kda.PATH_FUSED, _prefill(dict(inp, S0=S0), S_out=S0))
    assert S2.data_ptr() == S0.data_ptr()
    assert torch.equal(S2, S_ref) and torch.equal(o2, o_ref)


def test_fused_repeated_keys_full_replacement(cuda_device):
    """beta = 1, no decay, one repeated unit key: every output is a telescoping
    sum of corrected errors; the single pass keeps R and E at fp32 precision
    (bf16 hi + lo pairs), so the bf16 tolerance holds."""
    inp = W.make_prefill(1, 300, 2, 128, 128, "bf16", -3.0, 1.0, 0.0, seed=570, device=cuda_device)
    inp["k"][:] = inp["k"][:, :1]
    inp["beta"].fill_(1.0)
    inp["g"].zero_()
    o, S = _on_path(kda.PATH_FUSED, _prefill(inp))
    compare_units(inp, o, S, [(0, 0), (0, 1)], 1e-2)


def test_fused_workspace_is_small(cuda_device):
    kda.set_prefill_path(kda.PATH_FUSED)
    try:
        assert kda.workspace_size(8, 8192, 32, 128, 128, 0, 64, torch.bfloat16) <= 4096
        assert kda.workspace_size(1, 520998, 32, 128, 128, 16, 64, torch.bfloat16) <= 4096
        assert kda.prefill_phases(8, 8192, 32) == 1
    finally:
        kda.set_prefill_path(kda.PATH_AUTO)


def _repeated_key_input(B, T, H, seed, device):
    inp = W.make_prefill(B, T, H, 128, 128, "bf16", -3.0, 1.0, 0.0, seed=seed, device=device)
    inp["k"][:] = inp["k"][:, :1]
    inp["beta"].fill_(1.0)
    inp["g"].zero_()
    return inp


@pytest.mark.parametrize("segments", [0, 4])
def test_two_kernel_path_falls_back_on_near_parallel_keys(cuda_device, segments):
    """One repeated key makes every entry of A about 1: the two-kernel path's
    chunk-local kernels raise the fallback flag, its state pass stands down and
    the single-pass kernel recomputes the call, so the two-kernel call returns
    exactly the single pass's result (and meets the bf16 tolerance), with or
    without sequence segments."""
    inp = _repeated_key_input(1, 2048, 2, 571, cuda_device)
    kda.set_segment_chunks(segments if segments else -1)
    try:
        (o1, S1), (o2, S2) = _both_paths(_prefill(inp))
        if segments:
            assert kda.segment_chunks(1, 2048, 2) == segments
    finally:
        kda.set_segment_chunks(0)
    assert torch.equal(o1, o2) and torch.equal(S1, S2)
    compare_units(inp, o2, S2, [(0, 0), (0, 1)], 1e-2)


def test_two_kernel_path_keeps_its_own_result_on_ordinary_keys(cuda_device):
    """Random unit keys never reach |A| >= 0.5 here: the fallback stays idle and
    the two paths' (different) roundings give different bits."""
    inp = W.make_prefill(2, 512, 4, 128, 128, "bf16", -4.0, 1.0, 0.02, seed=572, device=cuda_device)
    (o1, S1), (o2, S2) = _both_paths(_prefill(inp))
    assert not torch.equal(o1, o2)
    assert rel_rms(o1.float().cpu().numpy(), o2.float().cpu().numpy()) < 1e-2


def test_single_pass_precise_instance_keeps_aliased_state(cuda_device):
    """The plain instance leaves a unit with near-parallel keys to the precise
    one without writing its state, so an S_out aliasing S0 still holds S0 when
    the precise instance starts from it."""
    inp = _repeated_key_input(2, 300, 2, 573, cuda_device)
    inp["S0"] = 0.05 * torch.randn((2, 2, 128, 128), generator=torch.Generator(device=cuda_device).manual_seed(5),
                                   device=cuda_device)
    o_ref, S_ref = _on_path(kda.PATH_FUSED, _prefill(inp))
    S0 = inp["S0"].clone()
    o2, S2 = _on_path(kda.PATH_FUSED, _prefill(dict(inp, S0=S0), S_out=S0))
    assert S2.data_ptr() == S0.data_ptr()
    assert torch.equal(o2, o_ref) and torch.equal(S2, S_ref)
    compare_units(inp, o_ref, S_ref, [(n, h) for n in range(2) for h in range(2)], 1e-2)


def test_single_pass_recomputes_only_marked_units(cuda_device):
    """Head 0 repeats one key (its unit is marked and recomputed by the precise
    instance), head 1 has random keys: head 1's result is bit for bit the one
    of a call in which no unit is marked."""
    rnd = W.make_prefill(1, 512, 2, 128, 128, "bf16", -3.0, 1.0, 0.0, seed=574, device=cuda_device)
    mixed = {k: (v.clone() if torch.is_tensor(v) else v) for k, v in rnd.items()}
    mixed["k"][:, :, 0] = mixed["k"][:, :1, 0]
    mixed["beta"][:, :, 0] = 1.0
    o_r, S_r = _on_path(kda.PATH_FUSED, _prefill(rnd))
    o_m, S_m = _on_path(kda.PATH_FUSED, _prefill(mixed))
    assert torch.equal(o_m[:, :, 1], o_r[:, :, 1]) and torch.equal(S_m[:, 1], S_r[:, 1])
    compare_units(mixed, o_m, S_m, [(0, 0), (0, 1)], 1e-2)


@pytest.mark.parametrize("path", ["single", "two"])
def test_packed_sequences_with_near_parallel_keys(cuda_device, path):
    """Packed sequences (an empty one, ragged tails) where two of them repeat
    one key: the single pass marks those units and its precise instance
    recomputes them; the two-kernel path hands the call to its fallback.
    Either way every unit meets the bf16 tolerance, and S_out may alias S0."""
    lens = (300, 0, 129, 64, 450)
    inp = W.make_prefill(1, sum(lens), 3, 128, 128, "bf16", -3.0, 1.0, 0.05, seed=575, device=cuda_device,
                         lengths=lens)
    cu = inp["cu_seqlens"]
    for seq in (0, 4):  # sequences 0 and 4: one key repeated over the whole sequence, beta = 1
        t0, t1 = int(cu[seq]), int(cu[seq + 1])
        inp["k"][:, t0:t1] = inp["k"][:, t0:t0 + 1]
        inp["beta"][:, t0:t1] = 1.0
    p = kda.PATH_FUSED if path == "single" else kda.PATH_TWO_KERNEL
    o_ref, S_ref = _on_path(p, _prefill(inp, cu))
    units = [(n, h) for n in range(len(lens)) for h in range(3)]
    compare_units(inp, o_ref, S_ref, units, 1e-2)
    S0 = inp["S0"].clone()
    o2, S2 = _on_path(p, _prefill(dict(inp, S0=S0), cu, S_out=S0))
    assert S2.data_ptr() == S0.data_ptr()
    assert torch.equal(o2, o_ref) and torch.equal(S2, S_ref)
