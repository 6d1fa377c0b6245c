"""CPU-side checks of the C ABI: libkda.so loads, exports every function that
include/kda.h declares, and rejects bad arguments before touching the GPU."""
import ctypes
import os
import re

import pytest

import kimi_delta_attention_31_b200 as kda

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "kda.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kda_[a-z_]+)\s*\(", src)))


def test_library_loads_and_exports_header_symbols():
    lib = kda.load_library()
    names = declared_functions()
    assert names, "no declarations parsed"
    assert set(names) == set(kda.EXPORTED)
    for n in names:
        assert hasattr(lib, n), n
    assert kda.version() == 100


def _null():
    return ctypes.c_void_p(0)


def _fake(addr=0x1000):
    return ctypes.c_void_p(addr)


def test_recurrent_step_rejects_bad_arguments():
    lib = kda.load_library()
    f = _fake()
    # unsupported head size
    st = lib.kda_recurrent_step(f, f, f, f, f, f, f, 4, 2, 96, 96, kda.KDA_BF16, None)
    assert st == 2 and "dk=96" in kda.last_error()
    # dk != dv
    st = lib.kda_recurrent_step(f, f, f, f, f, f, f, 4, 2, 128, 64, kda.KDA_BF16, None)
    assert st == 2
    # null pointer
    st = lib.kda_recurrent_step(f, f, _null(), f, f, f, f, 4, 2, 128, 128, kda.KDA_BF16, None)
    assert st == 1
    # misaligned pointers: the state must be 16-byte aligned, fp32 inputs 4-byte
    st = lib.kda_recurrent_step(f, f, f, f, f, _fake(0x1004), f, 4, 2, 64, 64, kda.KDA_F32, None)
    assert st == 3
    st = lib.kda_recurrent_step(f, f, _fake(0x1002), f, f, f, f, 4, 2, 64, 64, kda.KDA_F32, None)
    assert st == 3
    # bad dtype, bad sizes
    assert lib.kda_recurrent_step(f, f, f, f, f, f, f, 4, 2, 64, 64, 7, None) == 2
    assert lib.kda_recurrent_step(f, f, f, f, f, f, f, -1, 2, 64, 64, 0, None) == 1
    # nothing to do: N == 0 succeeds without launching
    assert lib.kda_recurrent_step(f, f, f, f, f, f, f, 0, 2, 64, 64, 0, None) == 0


def test_chunk_fwd_rejects_bad_arguments():
    lib = kda.load_library()
    f = _fake()
    args = lambda **kw: dict(dict(num_seqs=0, B=1, T=64, H=2, dk=128, dv=128, C=64, dt=0, cu=None,
                                  o=f, ws=None, wsb=0), **kw)

    def call(a):
        return lib.kda_chunk_fwd(f, f, f, f, f, None, a["o"], f, a["cu"], a["num_seqs"], a["B"], a["T"],
                                 a["H"], a["dk"], a["dv"], a["C"], a["dt"], a["ws"], a["wsb"], None)

    assert call(args(C=48)) == 2
    assert call(args(dk=80, dv=80)) == 2
    assert call(args(num_seqs=3)) == 1              # num_seqs without cu_seqlens
    assert call(args(cu=f, num_seqs=2, B=2)) == 1   # packed needs B == 1
    assert call(args(cu=f, num_seqs=0)) == 1
    assert call(args(o=_null())) == 1
    assert call(args(o=_fake(0x1008))) == 3
    assert call(args(H=0)) == 1
    assert call(args(dt=5)) == 2
    assert call(args(B=0)) == 0  # no sequences: nothing to do


def test_workspace_size_is_consistent():
    lib = kda.load_library()
    # fp32 arithmetic path needs no workspace
    assert lib.kda_chunk_fwd_workspace_size(1, 256, 2, 32, 32, 0, 16, kda.KDA_F32) == 0
    a = lib.kda_chunk_fwd_workspace_size(8, 8192, 32, 128, 128, 0, 64, kda.KDA_BF16)
    b = lib.kda_chunk_fwd_workspace_size(8, 8193, 32, 128, 128, 0, 64, kda.KDA_BF16)
    assert b >= a
    assert lib.kda_chunk_fwd_workspace_size(-1, 8, 2, 128, 128, 0, 64, kda.KDA_BF16) == 0


def test_binding_refuses_host_tensors():
    import torch
    x = torch.zeros(1, 4, 1, 32)
    with pytest.raises(ValueError):
        kda.chunk_fwd(x, x, x, x, torch.zeros(1, 4, 1))


def test_gdn_entry_points_validate_like_kda_with_a_per_token_gate():
    """kda_gdn_chunk_fwd takes g [B,T,H] (4-byte aligned is enough); the
    per-channel entry point keeps its 16-byte rule for g."""
    lib = kda.load_library()
    f = _fake()

    def call(fn, g, ws=None):
        return fn(f, f, f, g, f, None, _fake(0x2000), _fake(0x3000), None, 0, 1, 64, 2, 128, 128, 64,
                  kda.KDA_BF16, ws, 0, None)

    # both reach the workspace check (no workspace given) only if g passed
    assert call(lib.kda_gdn_chunk_fwd, _fake(0x1004)) == 4
    assert "kda_gdn_chunk_fwd" in kda.last_error()
    assert call(lib.kda_chunk_fwd, _fake(0x1004)) == 3
    assert call(lib.kda_gdn_chunk_fwd, _fake(0x1002)) == 3
    assert call(lib.kda_gdn_chunk_fwd, _null()) == 1
    st = lib.kda_gdn_recurrent_step(f, f, f, f, f, f, f, 4, 2, 96, 96, kda.KDA_BF16, None)
    assert st == 2 and kda.last_error().startswith("kda_gdn_recurrent_step")
    assert lib.kda_gdn_recurrent_step(f, f, f, _fake(0x1002), f, f, f, 4, 2, 64, 64, 0, None) == 3
    assert lib.kda_gdn_recurrent_step(f, f, f, f, f, f, f, 0, 2, 64, 64, 0, None) == 0


def test_binding_checks_gate_shapes():
    import torch
    x = torch.zeros(1, 4, 1, 32)
    # host tensors are refused before any shape logic; the shape rule is in the
    # message the binding raises for device tensors, checked on the GPU suite.
    with pytest.raises(ValueError):
        kda.gdn_chunk_fwd(x, x, x, torch.zeros(1, 4, 1), torch.zeros(1, 4, 1))


def test_prep_entry_points_validate_arguments():
    """kda_chunk_fwd_prep / kda_recurrent_step_prep: same checks as the plain
    entry points, plus the gate-logit dtype; the binding's signatures match."""
    lib = kda.load_library()
    f = _fake()

    def chunk(a, a_dt, ws=None):
        return lib.kda_chunk_fwd_prep(f, f, f, a, a_dt, f, None, _fake(0x2000), _fake(0x3000), None, 0, 1, 64,
                                      2, 128, 128, 64, kda.KDA_BF16, ws, 0, None)

    assert chunk(f, kda.KDA_BF16) == 4          # reached the workspace check
    assert "kda_chunk_fwd_prep" in kda.last_error()
    assert chunk(f, kda.KDA_F32) == 4
    assert chunk(f, 9) == 2                     # unknown logit dtype
    assert chunk(_fake(0x1008), kda.KDA_BF16) == 3  # logits need 16-byte alignment here
    assert chunk(_null(), kda.KDA_F32) == 1

    def step(a, a_dt, dk=64):
        return lib.kda_recurrent_step_prep(f, f, f, a, a_dt, f, f, f, 4, 2, dk, dk, kda.KDA_BF16, None)

    assert step(f, kda.KDA_BF16, dk=96) == 2
    assert kda.last_error().startswith("kda_recurrent_step_prep")
    assert step(_fake(0x1002), kda.KDA_BF16, dk=96) == 2   # shape is checked first
    assert step(f, 7) == 2
    assert lib.kda_recurrent_step_prep(f, f, f, f, kda.KDA_F32, f, f, f, 0, 2, 64, 64, 0, None) == 0


def test_selftest_bounded_wait_rejects_bad_limits():
    lib = kda.load_library()
    assert lib.kda_selftest_bounded_wait(0, None) == 1
    assert lib.kda_selftest_bounded_wait(2_000_000_000, None) == 1
    assert "limit_ns" in kda.last_error()


def test_chunk_bwd_validates_arguments():
    lib = kda.load_library()
    f = _fake()

    o1, o2, o3, o4 = _fake(0x7000), _fake(0x7100), _fake(0x7200), _fake(0x7300)

    def call(dtype=kda.KDA_BF16, d=128, dq=_fake(0x7400), ws=None, wsb=0, B=1, T=64, cu=None, ns=0, q=f):
        return lib.kda_chunk_bwd(q, f, f, f, f, None, f, None, dq, o1, o2, o3, o4, None, cu, ns, B, T, 2, d, d,
                                 dtype, ws, wsb, None)

    assert call() == 4                                # reached the workspace check
    assert "kda_chunk_bwd" in kda.last_error()
    assert call(d=96) == 2
    assert call(dtype=7) == 2
    assert call(dq=_null()) == 1
    assert call(dq=_fake(0x1002)) == 3                # fp32 gradients need 4-byte alignment
    assert call(q=_fake(0x1001)) == 3                 # bf16 inputs need 2-byte alignment
    assert call(cu=f, ns=0) == 1
    assert call(B=0) == 0
    # an output that aliases an input, or another output, is rejected
    g_ = _fake(0x5000)
    st = lib.kda_chunk_bwd(f, f, f, g_, _fake(0x5100), None, f, None, _fake(0x6000), _fake(0x6100), _fake(0x6200),
                           g_, _fake(0x6300), None, None, 0, 1, 64, 2, 128, 128, kda.KDA_BF16, None, 0, None)
    assert st == 1 and "alias" in kda.last_error()
    st = lib.kda_chunk_bwd(f, f, f, g_, _fake(0x5100), None, f, None, _fake(0x6000), _fake(0x6000), _fake(0x6200),
                           _fake(0x6400), _fake(0x6300), None, None, 0, 1, 64, 2, 128, 128, kda.KDA_BF16, None, 0, None)
    assert st == 1 and "alias" in kda.last_error()
    need = lib.kda_chunk_bwd_workspace_size(1, 64, 2, 128, 128, 0)
    assert need == 4 * 2 * 128 * 128 * 4              # 4 chunks of 16 tokens x 2 heads x fp32 states
    assert call(ws=_fake(0x4000), wsb=need - 1) == 4


def test_local_kernel_switch():
    """kda_set_local_kernel takes 0 (warp-specialised where it applies) or 1
    (two-CTA kernel); anything else is KDA_ERR_INVALID_ARG and leaves the
    setting unchanged.  The binding mirrors the setting per thread."""
    lib = kda.load_library()
    assert lib.kda_set_local_kernel(7) == 1
    assert "variant" in kda.last_error()
    kda.set_local_kernel(1)
    try:
        assert not kda.uses_ws_kernel()
        assert kda.chunk_fwd_kernel_sequence(2, 128, 4) == ["kda_fused_setup_kernel", "kda_tc_chunk_local_kernel",
                                                            "kda_tc_state_pass_kernel", "kda_fused_prefill_kernel"]
    finally:
        kda.set_local_kernel(0)
    assert kda.uses_ws_kernel("log_token") and kda.uses_ws_kernel("logit", packed=True)
    # the precise fallback's set-up kernel first, its single-pass kernel last
    assert kda.chunk_fwd_kernel_sequence(2, 128, 4) == ["kda_fused_setup_kernel", "kda_ws_chunk_local_kernel",
                                                        "kda_tc_chunk_local_kernel", "kda_tc_state_pass_kernel",
                                                        "kda_fused_prefill_kernel"]
    assert kda.chunk_fwd_kernel_sequence(1, 300, 4, num_seqs=3)[:2] == ["kda_fused_setup_kernel",
                                                                       "kda_ws_chunk_table_kernel"]
    with pytest.raises(ValueError):
        kda.uses_ws_kernel("per_head")


def test_noalloc_binding_checks_arguments_before_any_launch():
    """chunk_fwd_noalloc checks dtypes and shapes exactly as chunk_fwd does:
    the C ABI sees only pointers, so a wrong dtype or shape would otherwise be
    read past its end on the device.  These fail before any CUDA call."""
    import torch
    B, T, H, d = 1, 8, 2, 32
    q = torch.zeros(B, T, H, d, dtype=torch.bfloat16)
    g = torch.zeros(B, T, H, d)
    beta = torch.zeros(B, T, H)
    for fn in (kda.chunk_fwd, kda.chunk_fwd_noalloc):
        with pytest.raises(TypeError):
            fn(q, q, q, g.to(torch.bfloat16), beta)           # bf16 g
        with pytest.raises(ValueError):
            fn(q, q, q, g[..., 0].contiguous(), beta)          # g of shape [B,T,H]
        with pytest.raises(ValueError):
            fn(q, q, q, g, torch.zeros(B, T, H + 1))           # beta of the wrong shape
        with pytest.raises(TypeError):
            fn(q, q, q, g, beta, cu_seqlens=torch.tensor([0, T], dtype=torch.int64))
        with pytest.raises(ValueError):
            fn(q, q, q, g, beta)                               # right shapes, host tensors


def test_backward_bindings_check_the_gate_layout_before_any_launch():
    """chunk_bwd takes one gate per key channel and gdn_chunk_bwd one per token
    and head; the C ABI sees only pointers, so the bindings refuse the other
    layout (and a non-fp32 gate) before any CUDA call."""
    import torch
    B, T, H, d = 1, 8, 2, 32
    q = torch.zeros(B, T, H, d, dtype=torch.bfloat16)
    beta = torch.zeros(B, T, H)
    g_ch, g_tok = torch.zeros(B, T, H, d), torch.zeros(B, T, H)
    for fn, good, other in ((kda.chunk_bwd, g_ch, g_tok), (kda.gdn_chunk_bwd, g_tok, g_ch)):
        with pytest.raises(TypeError):
            fn(q, q, q, good.to(torch.bfloat16), beta, q)      # bf16 gate
        with pytest.raises(ValueError):
            fn(q, q, q, other, beta, q)                        # the other gate layout
        with pytest.raises(ValueError):
            fn(q, q, q, good, beta, q)                         # right shapes, host tensors
    a = torch.zeros(B, T, H, d, dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        kda.chunk_bwd_prep(q, q, q, a.to(torch.float16), beta, q)   # half-precision gate logits
    with pytest.raises(ValueError):
        kda.chunk_bwd_prep(q, q, q, a[..., 0].contiguous(), beta, q)  # a of shape [B,T,H]
    with pytest.raises(ValueError):
        kda.chunk_bwd_prep(q, q, q, a, beta, q)                   # right shapes, host tensors


def test_host_entry_point_sizes_and_argument_checks():
    """kda_chunk_fwd_host: its device buffer holds a copy of every tensor plus
    the workspace, and bad arguments are refused before any copy is queued."""
    lib = kda.load_library()
    B, T, H, d = 4, 96, 2, 64
    tensors = 2 * B * T * H * d * 4 + B * T * H * d * 4 + B * T * H * d * 4 + B * T * H * 4 + 2 * B * H * d * d * 4
    size = lib.kda_chunk_fwd_host_buffer_size(B, T, H, d, d, 0, 32, kda.KDA_F32, 2)
    assert size >= tensors
    assert lib.kda_chunk_fwd_host_buffer_size(B, T, H, 96, 96, 0, 32, kda.KDA_F32, 2) == 0
    assert lib.kda_chunk_fwd_host_buffer_size(B, T, H, d, d, 0, 32, kda.KDA_F32, 0) == 0
    f = _fake()

    def call(dk=d, buf=0x10000, nbytes=None, pieces=2):
        nb = size if nbytes is None else nbytes
        return lib.kda_chunk_fwd_host(f, f, f, f, f, None, f, f, None, 0, B, T, H, dk, dk, 32, kda.KDA_F32,
                                      pieces, ctypes.c_void_p(buf), nb, None, None, None)

    assert call(dk=80) == 2
    assert call(pieces=0) == 1
    assert call(buf=0x10010) == 3          # device buffer not 256-byte aligned
    assert call(nbytes=size - 1) == 4      # too small
    assert "kda_chunk_fwd_host" in kda.last_error()
