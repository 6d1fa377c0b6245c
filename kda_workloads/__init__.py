"""Seeded synthetic inputs for the KDA workloads.

This module is shared by the tests, the smoke check and the benchmark: it
draws the random inputs both the CUDA path and the fp64 oracle consume.  It
holds none of the recurrence's arithmetic.  The input recipe (which is part of
each workload's definition, not of the method) is:

* q, k ~ N(0, 1) in fp32, then L2-normalised per (token, head) over dk in
  fp32 ("Kimi K3 notes 1: KDA" section 4: q and k are L2-normalised feature
  vectors), then rounded to the workload dtype;
* v ~ N(0, 1), rounded to the workload dtype;
* beta = sigmoid(N(0, 1)) in fp32 (a write strength in (0, 1));
* g = log(alpha) = -softplus(N(mu, sigma)) in fp32 (alpha in (0, 1)), one per
  key channel, or one per token and head for the Gated DeltaNet workloads;
* S0 ~ N(0, s0_std^2) in fp32, or zeros.

Draw order is q, k, v, beta-logit, alpha-logit, S0 from one torch generator
seeded with the workload's seed, on the device the tensors are created on
(CPU here, CUDA on a GPU machine -- the two streams differ, so both sides of a
comparison always read the very same tensors).
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch
import torch.nn.functional as F


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    H: int
    dk: int
    dv: int
    dtype: str  # "bf16" or "f32": dtype of q, k, v, o
    g_mu: float
    g_sigma: float
    s0_std: float  # 0 => zero initial state
    chunk: int
    seed: int
    lengths: Optional[tuple] = None  # packed varlen sequence lengths (B == 1)
    scalar_gate: bool = False  # Gated DeltaNet: g is [B, T, H] (one gate per token and head)
    raw_a_dtype: Optional[str] = None  # raw projections for the fused-preparation entry points

    @property
    def tokens(self) -> int:
        return sum(self.lengths) if self.lengths else self.B * self.T

    @property
    def num_seqs(self) -> int:
        return len(self.lengths) if self.lengths else self.B

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32


def varlen_lengths(seed: int = 4004, n: int = 16, lo: int = 1024, hi: int = 65536,
                   total_lo: int = 480 * 1024, total_hi: int = 544 * 1024) -> tuple:
    """16 lengths uniform in [lo, hi]; redraw with seed+1 until the sum is in range."""
    s = seed
    while True:
        gen = torch.Generator().manual_seed(s)
        lens = torch.randint(lo, hi + 1, (n,), generator=gen).tolist()
        if total_lo <= sum(lens) <= total_hi:
            return tuple(int(x) for x in lens)
        s += 1


# The five workloads: oracle-sized fp32, bf16 prefill, the training-shape
# prefill the headline number is quoted on, long packed varlen prefill, and
# recurrent decode (256 sequences x 32 heads, 1024 steps).
ORACLE_SMALL = Workload("kda_fwd_f32_B1_H2_T256_d32", 1, 256, 2, 32, 32, "f32", -3.0, 1.0, 0.0, 16, 1000)
PREFILL_H16 = Workload("kda_prefill_bf16_B1_H16_T4096_d128", 1, 4096, 16, 128, 128, "bf16", -4.0, 1.0, 0.02, 64, 1001)
PREFILL_B8 = Workload("kda_prefill_bf16_B8_H32_T8192_d128", 8, 8192, 32, 128, 128, "bf16", -5.0, 1.5, 0.0, 64, 1002)
_VL = varlen_lengths()
PREFILL_VARLEN = Workload("kda_prefill_varlen_bf16_16seq_H32_d128", 1, sum(_VL), 32, 128, 128, "bf16",
                          -4.0, 1.0, 0.0, 64, 1003, lengths=_VL)
DECODE = Workload("kda_decode_bf16_N256_H32_d128_1024steps", 256, 1024, 32, 128, 128, "bf16",
                  -3.0, 1.0, 0.02, 1, 1004)
# Gated DeltaNet (scalar gate) on the shapes of the prefill headline and of decode.
GDN_PREFILL_B8 = Workload("gdn_prefill_bf16_B8_H32_T8192_d128", 8, 8192, 32, 128, 128, "bf16",
                          -5.0, 1.5, 0.0, 64, 1005, scalar_gate=True)
GDN_DECODE = Workload("gdn_decode_bf16_N256_H32_d128_1024steps", 256, 1024, 32, 128, 128, "bf16",
                      -3.0, 1.0, 0.02, 1, 1006, scalar_gate=True)

# The headline prefill shape from raw projections: unnormalised q, k, bf16 gate
# logits a (log alpha = -softplus(a)), fp32 beta logits b.
PREP_PREFILL_B8 = Workload("kda_prefill_prep_bf16logits_B8_H32_T8192_d128", 8, 8192, 32, 128, 128, "bf16",
                           -5.0, 1.5, 0.0, 64, 1007, raw_a_dtype="bf16")

# One long sequence with few heads: too few (sequence, head) units for the GPU,
# the case sequence segments exist for.
LONG_SEQ = Workload("kda_prefill_bf16_B1_H8_T131072_d128", 1, 131072, 8, 128, 128, "bf16",
                    -5.0, 1.5, 0.0, 64, 1008)

WORKLOADS = {w.name: w for w in (ORACLE_SMALL, PREFILL_H16, PREFILL_B8, PREFILL_VARLEN, DECODE,
                                 GDN_PREFILL_B8, GDN_DECODE, PREP_PREFILL_B8, LONG_SEQ)}


def cu_seqlens_of(lengths, device="cpu") -> torch.Tensor:
    cu = [0]
    for x in lengths:
        cu.append(cu[-1] + int(x))
    return torch.tensor(cu, dtype=torch.int32, device=device)


def _unit_rows(x: torch.Tensor) -> torch.Tensor:
    # L2 normalisation over the last axis, in fp32 (input recipe, see module doc)
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)


def make_prefill(B, T, H, dk, dv, dtype="bf16", g_mu=-4.0, g_sigma=1.0, s0_std=0.0,
                 seed=0, device="cpu", lengths=None, normalize_qk=True, scalar_gate=False) -> dict:
    """Prefill inputs.  With ``lengths`` the layout is packed (B must be 1,
    T = sum(lengths)) and ``cu_seqlens`` (int32) is included.  With
    ``scalar_gate`` g is [B, T, H] (Gated DeltaNet) instead of [B, T, H, dk]."""
    if lengths is not None:
        assert B == 1 and T == sum(lengths)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    gen = torch.Generator(device=device).manual_seed(seed)
    shp_k = (B, T, H, dk)
    shp_v = (B, T, H, dv)
    q = torch.randn(shp_k, generator=gen, device=device, dtype=torch.float32)
    k = torch.randn(shp_k, generator=gen, device=device, dtype=torch.float32)
    v = torch.randn(shp_v, generator=gen, device=device, dtype=torch.float32)
    b_logit = torch.randn((B, T, H), generator=gen, device=device, dtype=torch.float32)
    a_logit = torch.randn((B, T, H) if scalar_gate else shp_k, generator=gen, device=device,
                          dtype=torch.float32)
    N = len(lengths) if lengths is not None else B
    if s0_std > 0:
        S0 = torch.randn((N, H, dk, dv), generator=gen, device=device, dtype=torch.float32) * s0_std
    else:
        S0 = None
    if normalize_qk:
        q = _unit_rows(q)
        k = _unit_rows(k)
    out = dict(
        q=q.to(tdt).contiguous(),
        k=k.to(tdt).contiguous(),
        v=v.to(tdt).contiguous(),
        beta=torch.sigmoid(b_logit).contiguous(),
        g=(-F.softplus(a_logit * g_sigma + g_mu)).contiguous(),
        S0=S0,
    )
    if lengths is not None:
        out["cu_seqlens"] = cu_seqlens_of(lengths, device)
    return out


def make_prefill_raw(B, T, H, dk, dv, dtype="bf16", a_mu=-5.0, a_sigma=1.5, a_dtype="bf16",
                     s0_std=0.0, seed=0, device="cpu", lengths=None) -> dict:
    """Raw projections for the fused-preparation entry points.  Same draws and
    order as make_prefill (q, k, v, beta-logit, alpha-logit, S0), but q and k
    are not normalised, b is the beta logit itself and a = N(a_mu, a_sigma) is
    the gate logit (log alpha = -softplus(a)), rounded to ``a_dtype``."""
    if lengths is not None:
        assert B == 1 and T == sum(lengths)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    adt = torch.bfloat16 if a_dtype == "bf16" else torch.float32
    gen = torch.Generator(device=device).manual_seed(seed)
    q = torch.randn((B, T, H, dk), generator=gen, device=device, dtype=torch.float32)
    k = torch.randn((B, T, H, dk), generator=gen, device=device, dtype=torch.float32)
    v = torch.randn((B, T, H, dv), generator=gen, device=device, dtype=torch.float32)
    b = torch.randn((B, T, H), generator=gen, device=device, dtype=torch.float32)
    a = torch.randn((B, T, H, dk), generator=gen, device=device, dtype=torch.float32) * a_sigma + a_mu
    N = len(lengths) if lengths is not None else B
    S0 = (torch.randn((N, H, dk, dv), generator=gen, device=device, dtype=torch.float32) * s0_std
          if s0_std > 0 else None)
    out = dict(q=q.to(tdt).contiguous(), k=k.to(tdt).contiguous(), v=v.to(tdt).contiguous(),
               a=a.to(adt).contiguous(), b=b.contiguous(), S0=S0)
    if lengths is not None:
        out["cu_seqlens"] = cu_seqlens_of(lengths, device)
    return out


def make_workload(w: Workload, device="cpu") -> dict:
    if w.raw_a_dtype is not None:
        return make_prefill_raw(w.B, w.T, w.H, w.dk, w.dv, w.dtype, w.g_mu, w.g_sigma, w.raw_a_dtype,
                                w.s0_std, w.seed, device, lengths=w.lengths)
    return make_prefill(w.B, w.T, w.H, w.dk, w.dv, w.dtype, w.g_mu, w.g_sigma, w.s0_std,
                        w.seed, device, lengths=w.lengths, scalar_gate=w.scalar_gate)


def make_decode_state(N, H, dk, dv, s0_std=0.02, seed=0, device="cpu") -> torch.Tensor:
    gen = torch.Generator(device=device).manual_seed(seed)
    return torch.randn((N, H, dk, dv), generator=gen, device=device, dtype=torch.float32) * s0_std


def make_decode_steps(N, H, dk, dv, steps, dtype="bf16", g_mu=-3.0, g_sigma=1.0, seed=0,
                      device="cpu", scalar_gate=False) -> dict:
    """``steps`` consecutive single-token inputs: q, k, g [steps,N,H,dk], v [steps,N,H,dv],
    beta [steps,N,H]; q and k unit-norm per (step, seq, head).  With
    ``scalar_gate`` g is [steps,N,H] (Gated DeltaNet)."""
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    gen = torch.Generator(device=device).manual_seed(seed + 7919)
    q = _unit_rows(torch.randn((steps, N, H, dk), generator=gen, device=device))
    k = _unit_rows(torch.randn((steps, N, H, dk), generator=gen, device=device))
    v = torch.randn((steps, N, H, dv), generator=gen, device=device)
    b_logit = torch.randn((steps, N, H), generator=gen, device=device)
    a_logit = torch.randn((steps, N, H) if scalar_gate else (steps, N, H, dk), generator=gen, device=device)
    return dict(q=q.to(tdt).contiguous(), k=k.to(tdt).contiguous(), v=v.to(tdt).contiguous(),
                beta=torch.sigmoid(b_logit).contiguous(),
                g=(-F.softplus(a_logit * g_sigma + g_mu)).contiguous())


def bytes_of(*tensors) -> int:
    return int(sum(t.numel() * t.element_size() for t in tensors if t is not None))


def describe(w: Workload) -> str:
    sl = f", lengths={list(w.lengths)}" if w.lengths else ""
    gate = " per token and head" if w.scalar_gate else " per key channel"
    return (f"{w.name}: B={w.B} T={w.T} H={w.H} dk={w.dk} dv={w.dv} {w.dtype}; "
            f"log alpha=-softplus(N({w.g_mu},{w.g_sigma})){gate}; S0 std={w.s0_std}; C={w.chunk}{sl}")


__all__ = ["Workload", "WORKLOADS", "ORACLE_SMALL", "PREFILL_H16", "PREFILL_B8", "PREFILL_VARLEN",
           "DECODE", "GDN_PREFILL_B8", "GDN_DECODE", "PREP_PREFILL_B8", "LONG_SEQ", "make_prefill_raw", "make_prefill", "make_workload", "make_decode_state", "make_decode_steps",
           "cu_seqlens_of", "varlen_lengths", "bytes_of", "describe"]
