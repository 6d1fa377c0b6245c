"""GPU parity of the two chunk-local kernels of the two-kernel tensor-core
prefill (kda_set_prefill_path(2)): the warp-specialised one (its default) and
the two-CTA-per-SM one (kda_set_local_kernel(1)).
Both against the fp64 oracle, and against each other on the same inputs,
including launches where chunks past the single-reference decay range
(log-decay below -80 over the chunk on some channel) are mixed in at random,
so that the warp-specialised kernel hands a scattered subset of its items to
the two-CTA kernel's item lists.
"""
import pytest
import torch

import kimi_delta_attention_31_b200 as kda
import kda_workloads as W
from parity_util import compare_units, compare_units_prep, rel_rms

pytestmark = pytest.mark.gpu


def _both(inp):
    outs = []
    for variant in (0, 1):
        kda.set_local_kernel(variant)
        kda.set_prefill_path(kda.PATH_TWO_KERNEL)
        try:
            o, S = kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp.get("S0"), None, 64)
        finally:
            kda.set_local_kernel(0)
            kda.set_prefill_path(kda.PATH_AUTO)
        torch.cuda.synchronize()
        assert kda.device_error() == 0
        outs.append((o, S))
    return outs


def _steep_mix(inp, seed, frac):
    """Per (batch row, chunk, head): with probability `frac` a log-decay of
    about -1.5 per token (-96 over a full chunk), else about -0.05."""
    B, T, H, dk = inp["g"].shape
    dev = inp["g"].device
    gen = torch.Generator(device=dev).manual_seed(seed)
    nc = (T + 63) // 64
    steep = torch.rand((B, nc, H), generator=gen, device=dev) < frac
    rate = torch.where(steep, torch.full_like(steep, 1.5, dtype=torch.float32),
                       torch.full_like(steep, 0.05, dtype=torch.float32))
    rate = rate.repeat_interleave(64, dim=1)[:, :T]  # [B, T, H]
    u = torch.rand(inp["g"].shape, generator=gen, device=dev)
    inp["g"] = (-rate.unsqueeze(-1) * (1.0 - 0.005 * u)).contiguous()
    return int(steep.sum())


@pytest.mark.parametrize("B,T,H", [(1, 1, 1), (1, 64, 2), (2, 200, 4), (3, 130, 3), (2, 1000, 5)])
def test_local_kernels_agree(cuda_device, B, T, H):
    inp = W.make_prefill(B, T, H, 128, 128, "bf16", -4.0, 1.0, 0.05, seed=300 + T + H, device=cuda_device)
    (o0, S0), (o1, S1) = _both(inp)
    units = [(n, h) for n in range(B) for h in range(H)]
    compare_units(inp, o0, S0, units, 1e-2)
    compare_units(inp, o1, S1, units, 1e-2)
    assert rel_rms(o0.float().cpu(), o1.float().cpu()) < 1e-3
    assert rel_rms(S0.cpu(), S1.cpu()) < 1e-3


@pytest.mark.parametrize("frac", [0.1, 0.5, 0.9])
def test_local_kernels_scattered_steep_chunks(cuda_device, frac):
    """B4 T2048 H8: 1024 items, about 7 per CTA of the warp-specialised kernel,
    a random subset of them steep."""
    inp = W.make_prefill(4, 2048, 8, 128, 128, "bf16", -4.0, 1.0, 0.05, seed=41, device=cuda_device)
    n_steep = _steep_mix(inp, seed=42 + int(frac * 10), frac=frac)
    assert 0 < n_steep < 4 * 32 * 8
    (o0, S0), (o1, S1) = _both(inp)
    assert torch.isfinite(o0).all() and torch.isfinite(S0).all()
    units = [(0, 0), (1, 3), (2, 5), (3, 7), (3, 1)]
    compare_units(inp, o0, S0, units, 1e-2)
    assert rel_rms(o0.float().cpu(), o1.float().cpu()) < 1e-3
    assert rel_rms(S0.cpu(), S1.cpu()) < 1e-3


def _both_fn(fn):
    outs = []
    for variant in (0, 1):
        kda.set_local_kernel(variant)
        kda.set_prefill_path(kda.PATH_TWO_KERNEL)
        try:
            o, S = fn()
        finally:
            kda.set_local_kernel(0)
            kda.set_prefill_path(kda.PATH_AUTO)
        torch.cuda.synchronize()
        assert kda.device_error() == 0
        outs.append((o, S))
    return outs


@pytest.mark.parametrize("B,T,H", [(1, 64, 2), (2, 200, 4), (2, 1000, 5)])
def test_local_kernels_agree_gdn(cuda_device, B, T, H):
    """Per-token gate (Gated DeltaNet): the warp-specialised kernel reads it
    with plain loads (no tensor copy)."""
    inp = W.make_prefill(B, T, H, 128, 128, "bf16", -3.0, 1.0, 0.05, seed=340 + T, device=cuda_device,
                         scalar_gate=True)
    (o0, S0), (o1, S1) = _both_fn(lambda: kda.gdn_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                                            inp["S0"], None, 64))
    units = [(n, h) for n in range(B) for h in range(H)]
    compare_units(inp, o0, S0, units, 1e-2)
    assert rel_rms(o0.float().cpu(), o1.float().cpu()) < 1e-3
    assert rel_rms(S0.cpu(), S1.cpu()) < 1e-3


@pytest.mark.parametrize("a_dtype", ["f32", "bf16"])
@pytest.mark.parametrize("B,T,H", [(1, 65, 2), (2, 1000, 5)])
def test_local_kernels_agree_prep(cuda_device, a_dtype, B, T, H):
    """Raw projections: q, k normalised, -softplus of the gate logits and the
    sigmoid of beta's logits inside the kernels."""
    inp = W.make_prefill_raw(B, T, H, 128, 128, "bf16", -3.0, 1.0, a_dtype, 0.05, seed=360 + T,
                             device=cuda_device)
    (o0, S0), (o1, S1) = _both_fn(lambda: kda.chunk_fwd_prep(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"],
                                                             inp["S0"], None, 64))
    compare_units_prep(inp, o0, S0, [(n, h) for n in range(B) for h in range(H)], 1e-2)
    assert rel_rms(o0.float().cpu(), o1.float().cpu()) < 1e-3
    assert rel_rms(S0.cpu(), S1.cpu()) < 1e-3


@pytest.mark.parametrize("lens", [(0, 1, 17, 64, 65, 100, 3), (130,) * 40 + (0, 7), (4096, 1, 2000, 64)])
def test_local_kernels_agree_packed(cuda_device, lens):
    """Packed sequences (cu_seqlens): the warp-specialised kernel looks chunk
    positions up in a table a one-CTA kernel builds from cu_seqlens, and stops
    at the exact chunk count read on the device (the host's item count is an
    upper bound)."""
    inp = W.make_prefill(1, sum(lens), 3, 128, 128, "bf16", -4.0, 1.0, 0.05, seed=380 + len(lens),
                         device=cuda_device, lengths=lens)
    (o0, S0), (o1, S1) = _both_fn(lambda: kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                                        inp["S0"], inp["cu_seqlens"], 64))
    units = [(n, h) for n in range(len(lens)) for h in range(3)][:24]
    compare_units(inp, o0, S0, units, 1e-2)
    assert rel_rms(o0.float().cpu(), o1.float().cpu()) < 1e-3
    assert rel_rms(S0.cpu(), S1.cpu()) < 1e-3
    for n, L in enumerate(lens):  # an empty sequence hands its state through
        if L == 0:
            assert torch.equal(S0[n], inp["S0"][n])


def test_local_kernels_packed_steep_mix(cuda_device):
    """Packed sequences with steep chunks mixed in: the item lists hold
    packed-layout items that the two-CTA kernel locates from cu_seqlens."""
    lens = (700, 64, 1000, 5, 300)
    inp = W.make_prefill(1, sum(lens), 4, 128, 128, "bf16", -4.0, 1.0, 0.05, seed=391, device=cuda_device,
                         lengths=lens)
    gen = torch.Generator(device=cuda_device).manual_seed(392)
    # sequences 0 and 2 decay by about -1.5 per token (-96 over a full chunk:
    # past the single-reference range), the others by about -0.05
    rate = torch.cat([torch.full((L,), 1.5 if n in (0, 2) else 0.05) for n, L in enumerate(lens)])
    rate = rate.to(cuda_device).view(1, -1, 1, 1)
    inp["g"] = (-rate * (1.0 - 0.005 * torch.rand(inp["g"].shape, generator=gen, device=cuda_device))).contiguous()
    (o0, S0), (o1, S1) = _both_fn(lambda: kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                                        inp["S0"], inp["cu_seqlens"], 64))
    assert torch.isfinite(o0).all() and torch.isfinite(S0).all()
    compare_units(inp, o0, S0, [(0, 0), (1, 1), (2, 2), (3, 3), (4, 0)], 1e-2)
    assert rel_rms(o0.float().cpu(), o1.float().cpu()) < 1e-3
    assert rel_rms(S0.cpu(), S1.cpu()) < 1e-3
