"""GPU parity of the backward pass (kda_chunk_bwd; kda_gdn_chunk_bwd for one
gate per token and head; kda_chunk_bwd_prep from raw projections) against
the gradient oracle (reverse-mode
differentiation of the fp64 token recurrence).  The
kernel computes in fp32 from the same (bf16- or fp32-rounded) inputs the
oracle widens, so both dtypes are held to 1e-4 relative RMS per (sequence,
head) slice of every gradient."""
import numpy as np
import pytest
import torch

import kimi_delta_attention_31_b200 as kda
import kda_workloads as W
from oracle.grad import gdn_recurrent_grad, recurrent_grad, recurrent_prep_grad
from parity_util import rel_rms

pytestmark = pytest.mark.gpu

TOL = 1e-4


def _inputs(dev, B, T, H, d, dtype, seed, lengths=None, s0=True, scalar_gate=False):
    inp = W.make_prefill(B, T, H, d, d, dtype, -3.0, 1.0, 0.05 if s0 else 0.0, seed=seed, device=dev, lengths=lengths,
                         scalar_gate=scalar_gate)
    gen = torch.Generator(device=dev).manual_seed(seed + 1)
    tdt = inp["q"].dtype
    inp["do"] = torch.randn(inp["v"].shape, generator=gen, device=dev).to(tdt)
    N = len(lengths) if lengths else B
    inp["dS_T"] = torch.randn((N, H, d, d), generator=gen, device=dev) * 0.1
    return inp


def _check_slices(got, ref, what, tol=TOL):
    """got, ref: [..] arrays with the (sequence, head) slice structure of the tensor."""
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    err = rel_rms(got, ref)
    assert err <= tol, f"{what}: rel-RMS {err:.3e}"
    return err


def _compare(inp, out, with_s0=True, grad=recurrent_grad):
    cpu = {n: (t.double().cpu().numpy() if t is not None else None) for n, t in inp.items() if n != "cu_seqlens"}
    B, T, H, d = cpu["q"].shape
    for b in range(B):
        for h in range(H):
            sl = lambda x: x[b:b + 1, :, h:h + 1]
            ref = grad(sl(cpu["q"]), sl(cpu["k"]), sl(cpu["v"]), sl(cpu["g"]), sl(cpu["beta"]),
                                 cpu["S0"][b:b + 1, h:h + 1] if with_s0 else None, sl(cpu["do"]),
                                 cpu["dS_T"][b:b + 1, h:h + 1])
            for n in ("dq", "dk", "dv", "dg", "dbeta"):
                _check_slices(out[n][b:b + 1, :, h:h + 1].double().cpu().numpy(), ref[n], f"{n} b{b} h{h}")
            if with_s0:
                _check_slices(out["dS0"][b:b + 1, h:h + 1].double().cpu().numpy(), ref["dS0"], f"dS0 b{b} h{h}")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("T", [1, 17, 40])
def test_bwd_small_shapes(cuda_device, dtype, d, T):
    inp = _inputs(cuda_device, 2, T, 2, d, dtype, seed=600 + T + d)
    out = kda.chunk_bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["do"], inp["S0"], inp["dS_T"])
    torch.cuda.synchronize()
    _compare(inp, out)


def test_bwd_zero_initial_state_and_no_final_gradient(cuda_device):
    inp = _inputs(cuda_device, 1, 33, 2, 64, "bf16", seed=61, s0=False)
    out = kda.chunk_bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["do"], None, None, need_dS0=False)
    torch.cuda.synchronize()
    inp["dS_T"] = torch.zeros_like(inp["dS_T"])
    _compare(inp, out, with_s0=False)


def test_bwd_packed_varlen(cuda_device):
    lens = (5, 0, 33, 16)
    inp = _inputs(cuda_device, 1, sum(lens), 2, 64, "f32", seed=62, lengths=lens)
    out = kda.chunk_bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["do"], inp["S0"], inp["dS_T"],
                        cu_seqlens=inp["cu_seqlens"])
    torch.cuda.synchronize()
    cu = np.cumsum((0,) + lens)
    cpu = {n: t.double().cpu().numpy() for n, t in inp.items() if n not in ("cu_seqlens",)}
    for s_i in range(len(lens)):
        a, b = cu[s_i], cu[s_i + 1]
        for h in range(2):
            if b == a:  # empty sequence: the state gradient passes through
                assert torch.allclose(out["dS0"][s_i, h], inp["dS_T"][s_i, h])
                continue
            sl = lambda x: x[:, a:b, h:h + 1]
            ref = recurrent_grad(sl(cpu["q"]), sl(cpu["k"]), sl(cpu["v"]), sl(cpu["g"]), sl(cpu["beta"]),
                                 cpu["S0"][s_i:s_i + 1, h:h + 1], sl(cpu["do"]), cpu["dS_T"][s_i:s_i + 1, h:h + 1])
            for n in ("dq", "dk", "dv", "dg", "dbeta"):
                _check_slices(out[n][:, a:b, h:h + 1].double().cpu().numpy(), ref[n], f"{n} seq{s_i} h{h}")
            _check_slices(out["dS0"][s_i:s_i + 1, h:h + 1].double().cpu().numpy(), ref["dS0"], f"dS0 seq{s_i}")


def test_bwd_longer_sequence_strong_decay(cuda_device):
    """T = 300 at d = 128 with steep gates (log alpha about -2 per token): the
    backward uses only decay factors <= 1, so any gate is exact."""
    inp = _inputs(cuda_device, 1, 300, 1, 128, "bf16", seed=63)
    inp["g"] = (inp["g"] * 0 - 2.0 + 0.1 * torch.rand_like(inp["g"])).contiguous()
    out = kda.chunk_bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["do"], inp["S0"], inp["dS_T"])
    torch.cuda.synchronize()
    _compare(inp, out)


# ---- Gated DeltaNet (one gate per token and head)

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [32, 128])
@pytest.mark.parametrize("T", [17, 40])
def test_gdn_bwd_small_shapes(cuda_device, dtype, d, T):
    inp = _inputs(cuda_device, 2, T, 2, d, dtype, seed=700 + T + d, scalar_gate=True)
    out = kda.gdn_chunk_bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["do"], inp["S0"], inp["dS_T"])
    torch.cuda.synchronize()
    assert kda.device_error() == 0
    assert tuple(out["dg"].shape) == tuple(inp["g"].shape)
    _compare(inp, out, grad=gdn_recurrent_grad)


def test_gdn_bwd_packed_varlen(cuda_device):
    lens = (5, 0, 33, 16)
    inp = _inputs(cuda_device, 1, sum(lens), 2, 64, "f32", seed=72, lengths=lens, scalar_gate=True)
    out = kda.gdn_chunk_bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["do"], inp["S0"],
                            inp["dS_T"], cu_seqlens=inp["cu_seqlens"])
    torch.cuda.synchronize()
    cu = np.cumsum((0,) + lens)
    cpu = {n: t.double().cpu().numpy() for n, t in inp.items() if n not in ("cu_seqlens",)}
    for s_i in range(len(lens)):
        a, b = cu[s_i], cu[s_i + 1]
        for h in range(2):
            if b == a:  # empty sequence: the state gradient passes through
                assert torch.allclose(out["dS0"][s_i, h], inp["dS_T"][s_i, h])
                continue
            sl = lambda x: x[:, a:b, h:h + 1]
            ref = gdn_recurrent_grad(sl(cpu["q"]), sl(cpu["k"]), sl(cpu["v"]), sl(cpu["g"]), sl(cpu["beta"]),
                                     cpu["S0"][s_i:s_i + 1, h:h + 1], sl(cpu["do"]), cpu["dS_T"][s_i:s_i + 1, h:h + 1])
            for n in ("dq", "dk", "dv", "dg", "dbeta"):
                _check_slices(out[n][:, a:b, h:h + 1].double().cpu().numpy(), ref[n], f"{n} seq{s_i} h{h}")
            _check_slices(out["dS0"][s_i:s_i + 1, h:h + 1].double().cpu().numpy(), ref["dS0"], f"dS0 seq{s_i}")


def test_gdn_bwd_equals_the_per_channel_bwd_on_the_repeated_gate(cuda_device):
    """The scalar-gate backward reads the one gate where the per-channel one
    reads its copies and does the same arithmetic, so every gradient but dg
    agrees to fp32 rounding; dg is the per-channel dg summed over channels
    (up to fp32 summation order)."""
    inp = _inputs(cuda_device, 2, 70, 3, 64, "bf16", seed=73, scalar_gate=True)
    g_full = inp["g"][..., None].expand(*inp["g"].shape, 64).contiguous()
    out = kda.gdn_chunk_bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["do"], inp["S0"], inp["dS_T"])
    ref = kda.chunk_bwd(inp["q"], inp["k"], inp["v"], g_full, inp["beta"], inp["do"], inp["S0"], inp["dS_T"])
    torch.cuda.synchronize()
    for n in ("dq", "dk", "dv", "dbeta", "dS0"):
        assert rel_rms(out[n].double().cpu().numpy(), ref[n].double().cpu().numpy()) <= 1e-6, n
    err = rel_rms(out["dg"].double().cpu().numpy(), ref["dg"].sum(-1).double().cpu().numpy())
    assert err <= 1e-6, err


# ---- from raw projections (q, k unnormalised; gate and beta logits)

def _raw(dev, B, T, H, d, dtype, a_dtype, seed, lengths=None):
    inp = W.make_prefill_raw(B, T, H, d, d, dtype, -5.0, 1.5, a_dtype, 0.05, seed=seed, device=dev, lengths=lengths)
    gen = torch.Generator(device=dev).manual_seed(seed + 1)
    inp["do"] = torch.randn(inp["v"].shape, generator=gen, device=dev).to(inp["q"].dtype)
    N = len(lengths) if lengths else B
    inp["dS_T"] = torch.randn((N, H, d, d), generator=gen, device=dev) * 0.1
    return inp


def _compare_prep(inp, out, seqs):
    """seqs: list of (batch row, token range) per sequence."""
    cpu = {n: t.double().cpu().numpy() for n, t in inp.items() if n != "cu_seqlens" and t is not None}
    H = cpu["q"].shape[2]
    for s_i, (b, a0, a1) in enumerate(seqs):
        for h in range(H):
            sl = lambda x: x[b:b + 1, a0:a1, h:h + 1]
            ref = recurrent_prep_grad(sl(cpu["q"]), sl(cpu["k"]), sl(cpu["v"]), sl(cpu["a"]), sl(cpu["b"]),
                                      cpu["S0"][s_i:s_i + 1, h:h + 1], sl(cpu["do"]), cpu["dS_T"][s_i:s_i + 1, h:h + 1])
            for n in ("dq", "dk", "dv", "da", "db"):
                _check_slices(out[n][b:b + 1, a0:a1, h:h + 1].double().cpu().numpy(), ref[n], f"{n} seq{s_i} h{h}")
            _check_slices(out["dS0"][s_i:s_i + 1, h:h + 1].double().cpu().numpy(), ref["dS0"], f"dS0 seq{s_i}")


@pytest.mark.parametrize("dtype,a_dtype,d,T", [("f32", "f32", 64, 40), ("bf16", "bf16", 64, 40),
                                               ("bf16", "f32", 32, 17), ("bf16", "bf16", 128, 33)])
def test_prep_bwd_matches_the_oracle(cuda_device, dtype, a_dtype, d, T):
    inp = _raw(cuda_device, 2, T, 2, d, dtype, a_dtype, seed=800 + d + T)
    out = kda.chunk_bwd_prep(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"], inp["do"], inp["S0"], inp["dS_T"])
    torch.cuda.synchronize()
    assert kda.device_error() == 0
    _compare_prep(inp, out, [(b, 0, T) for b in range(2)])


def test_prep_bwd_packed_and_a_zero_query_row(cuda_device):
    """Packed sequences (one empty), and one token whose q is all zeros: its
    norm is clamped at 1e-12, where the normalisation is linear."""
    lens = (9, 0, 40, 16)
    inp = _raw(cuda_device, 1, sum(lens), 2, 64, "f32", "f32", seed=81, lengths=lens)
    inp["q"][0, 3, 1].zero_()
    out = kda.chunk_bwd_prep(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"], inp["do"], inp["S0"], inp["dS_T"],
                             cu_seqlens=inp["cu_seqlens"])
    torch.cuda.synchronize()
    cu = np.cumsum((0,) + lens)
    for s_i in range(len(lens)):
        if lens[s_i] == 0:
            assert torch.allclose(out["dS0"][s_i], inp["dS_T"][s_i])
    seqs = [(0, cu[i], cu[i + 1]) for i in range(len(lens))]
    keep = [i for i in range(len(lens)) if lens[i] > 0]
    sub = dict(inp)
    sub["S0"], sub["dS_T"] = inp["S0"][keep], inp["dS_T"][keep]
    out_sub = dict(out)
    out_sub["dS0"] = out["dS0"][keep]
    _compare_prep(sub, out_sub, [seqs[i] for i in keep])
