"""kda_chunk_fwd_noalloc: the prefill for callers that cannot allocate device
memory (for example a plug-in handed only input and output pointers by a host
framework that owns the device memory pool).  It runs the very same kernels as
kda_chunk_fwd with a caller-allocated workspace (without the automatic
sequence segments where their maps would not fit its array), so its results
must be bit-for-bit the same, call after call (its built-in scratch array is reused
and keeps the previous call's contents); it must refuse sizes its array cannot
hold and check its arguments exactly as chunk_fwd does.

This file is named so that pytest collects it last."""
import pytest
import torch

import kimi_delta_attention_31_b200 as kda
import kda_workloads as W

pytestmark = pytest.mark.gpu


def _same(x, ref_o, ref_S, o, S):
    assert torch.isfinite(o.float()).all() and torch.isfinite(S).all()
    assert torch.equal(o, ref_o) and torch.equal(S, ref_S)


def _both(x, cu=None, C=64):
    ref_o, ref_S = kda.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], cu, C)
    o, S = kda.chunk_fwd_noalloc(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], cu, C)
    torch.cuda.synchronize()
    return ref_o, ref_S, o, S


def test_noalloc_matches_workspace_entry_point_twice(cuda_device):
    # tensor-core shape (bf16, d=128, C=64), ragged last chunk, random initial state
    for seed in (901, 902):
        x = W.make_prefill(2, 700, 8, 128, 128, "bf16", -4.0, 1.0, 0.02, seed=seed, device=cuda_device)
        _same(x, *_both(x))


def test_noalloc_packed_sequences(cuda_device):
    lens = (64, 1, 130, 0, 77)
    x = W.make_prefill(1, sum(lens), 4, 128, 128, "bf16", -4.0, 1.0, 0.02, seed=903, device=cuda_device,
                       lengths=lens)
    _same(x, *_both(x, x["cu_seqlens"]))


def test_noalloc_at_its_documented_limit(cuda_device):
    # the two-kernel path keeps a per-chunk image: B=1, H=8, T=7168 (112 chunks x
    # 8 heads) is the largest case kda.h names for it.  Its automatic sequence
    # segments add state maps; where those would not fit the array, the
    # no-alloc call runs without them, so the reference runs the same way.
    sizes = (1, 7168, 8, 128, 128, 0, 64, torch.bfloat16)
    kda.set_prefill_path(kda.PATH_TWO_KERNEL)
    try:
        need_auto = kda.workspace_size(*sizes)
        kda.set_segment_chunks(-1)
        need_plain = kda.workspace_size(*sizes)
        assert 0 < need_plain <= kda.NOALLOC_SCRATCH_BYTES
        x = W.make_prefill(1, 7168, 8, 128, 128, "bf16", -4.0, 1.0, 0.02, seed=905, device=cuda_device)
        kda.set_segment_chunks(-1 if need_auto > kda.NOALLOC_SCRATCH_BYTES else 0)
        ref_o, ref_S = kda.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], None, 64)
        kda.set_segment_chunks(0)  # the no-alloc call decides for itself
        o, S = kda.chunk_fwd_noalloc(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], None, 64)
        torch.cuda.synchronize()
        _same(x, ref_o, ref_S, o, S)
        assert kda.device_error() == 0
    finally:
        kda.set_segment_chunks(0)
        kda.set_prefill_path(kda.PATH_AUTO)


def test_noalloc_single_pass_at_the_benchmark_size(cuda_device):
    # the single-pass prefill needs only a unit counter: B8 H32 T8192 fits easily
    kda.set_prefill_path(kda.PATH_FUSED)
    try:
        assert kda.workspace_size(8, 8192, 32, 128, 128, 0, 64, torch.bfloat16) <= 4096
        x = W.make_prefill(8, 8192, 32, 128, 128, "bf16", -5.0, 1.5, 0.0, seed=907, device=cuda_device)
        _same(x, *_both(x))
    finally:
        kda.set_prefill_path(kda.PATH_AUTO)


def test_noalloc_fp32_path_needs_no_scratch(cuda_device):
    assert kda.workspace_size(2, 100, 3, 64, 64, 0, 32, torch.float32) == 0
    x = W.make_prefill(2, 100, 3, 64, 64, "f32", -3.0, 1.0, 0.05, seed=906, device=cuda_device)
    _same(x, *_both(x, None, 32))


def test_noalloc_rejects_sizes_beyond_its_array(cuda_device):
    need = kda.workspace_size(1, 8192, 16, 128, 128, 0, 64, torch.bfloat16)
    assert need > kda.NOALLOC_SCRATCH_BYTES
    x = W.make_prefill(1, 8192, 16, 128, 128, "bf16", seed=904, device=cuda_device)
    with pytest.raises(kda.KDAError) as err:
        kda.chunk_fwd_noalloc(x["q"], x["k"], x["v"], x["g"], x["beta"])
    assert err.value.status == 4 and "built-in" in str(err.value)
