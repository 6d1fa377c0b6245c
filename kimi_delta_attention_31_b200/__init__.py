"""KDA (Kimi Delta Attention) on NVIDIA B200: Python binding of libkda.

Argument marshalling only: every step of the recurrence runs in the CUDA
kernels of ``libkda.so`` (declared in ``include/kda.h``).  PyTorch supplies
device memory and the current stream.  There is no CPU fallback: if the
library is missing, importing the binding's functions raises.

Public API
----------
chunk_fwd(q, k, v, g, beta, S0=None, cu_seqlens=None, chunk_size=64, ...)
    chunkwise prefill -> (o, S_out)
recurrent_step(q, k, v, g, beta, S, o=None)
    one decode token per sequence, S updated in place -> o
chunk_fwd_host(...)
    chunk_fwd for pinned host tensors: copies in, runs, copies results out
workspace_size(...), last_error(), device_error(), lib_path()
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libkda.so")
_lock = threading.Lock()
_lib = None

KDA_OK = 0
_STATUS = {0: "KDA_OK", 1: "KDA_ERR_INVALID_ARG", 2: "KDA_ERR_UNSUPPORTED", 3: "KDA_ERR_ALIGNMENT",
           4: "KDA_ERR_WORKSPACE", 5: "KDA_ERR_CUDA", 6: "KDA_ERR_DEVICE_TIMEOUT"}
KDA_BF16, KDA_F32 = 0, 1

# Every symbol include/kda.h declares (checked by the CPU test-suite).
EXPORTED = ("kda_chunk_fwd_workspace_size", "kda_chunk_fwd", "kda_recurrent_step",
            "kda_last_error", "kda_device_error", "kda_chunk_fwd_launches", "kda_profile_events",
            "kda_version", "kda_chunk_fwd_noalloc", "kda_gdn_chunk_fwd", "kda_gdn_recurrent_step",
            "kda_chunk_fwd_prep", "kda_recurrent_step_prep", "kda_selftest_bounded_wait",
            "kda_set_segment_chunks", "kda_segment_chunks", "kda_chunk_bwd", "kda_chunk_bwd_workspace_size",
            "kda_set_local_kernel", "kda_chunk_fwd_host", "kda_chunk_fwd_host_buffer_size",
            "kda_set_prefill_path", "kda_chunk_fwd_phases", "kda_gdn_chunk_bwd", "kda_chunk_bwd_prep",
            "kda_chunk_bwd_prep_workspace_size")
NOALLOC_SCRATCH_BYTES = 64 * 1024 * 1024

# Kernels of one kda_chunk_fwd call, in launch order, per path.
KERNELS_SIMT = ("kda_chunk_simt_kernel",)
KERNELS_TC = ("kda_tc_chunk_local_kernel", "kda_tc_state_pass_kernel")
KERNEL_WS = "kda_ws_chunk_local_kernel"
KERNEL_FUSED = "kda_fused_prefill_kernel"
PATH_AUTO, PATH_FUSED, PATH_TWO_KERNEL = 0, 1, 2
_tls = threading.local()  # mirrors kda_set_local_kernel / kda_set_prefill_path, which are per host thread


class KDAError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"{_STATUS.get(status, status)}: {msg}")
        self.status = status


def lib_path() -> str:
    return _LIB_PATH


def load_library():
    """Load libkda.so (building it first if the sources are newer).  Raises if
    it cannot be built or loaded: there is deliberately no fallback."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        from . import build as _build
        if _build.needs_build():
            _build.build()
        if not os.path.exists(_LIB_PATH):
            raise ImportError(f"libkda.so not found at {_LIB_PATH}; run "
                              "python -m kimi_delta_attention_31_b200.build")
        lib = ctypes.CDLL(_LIB_PATH)
        vp, i32, szt = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        lib.kda_chunk_fwd_workspace_size.argtypes = [i32] * 7 + [i32]
        lib.kda_chunk_fwd_workspace_size.restype = szt
        lib.kda_chunk_fwd.argtypes = [vp] * 9 + [i32] * 7 + [i32, vp, szt, vp]
        lib.kda_chunk_fwd.restype = i32
        lib.kda_recurrent_step.argtypes = [vp] * 7 + [i32] * 5 + [vp]
        lib.kda_recurrent_step.restype = i32
        lib.kda_gdn_chunk_fwd.argtypes = lib.kda_chunk_fwd.argtypes
        lib.kda_gdn_chunk_fwd.restype = i32
        lib.kda_gdn_recurrent_step.argtypes = lib.kda_recurrent_step.argtypes
        lib.kda_gdn_recurrent_step.restype = i32
        lib.kda_chunk_fwd_prep.argtypes = [vp] * 4 + [i32] + [vp] * 5 + [i32] * 7 + [i32, vp, szt, vp]
        lib.kda_chunk_fwd_prep.restype = i32
        lib.kda_recurrent_step_prep.argtypes = [vp] * 4 + [i32] + [vp] * 3 + [i32] * 5 + [vp]
        lib.kda_recurrent_step_prep.restype = i32
        lib.kda_last_error.argtypes = []
        lib.kda_last_error.restype = ctypes.c_char_p
        lib.kda_device_error.argtypes = [ctypes.POINTER(ctypes.c_int), vp]
        lib.kda_device_error.restype = i32
        lib.kda_chunk_fwd_launches.argtypes = [i32] * 4
        lib.kda_chunk_fwd_launches.restype = i32
        lib.kda_profile_events.argtypes = [vp, i32]
        lib.kda_profile_events.restype = i32
        lib.kda_chunk_fwd_host_buffer_size.argtypes = [i32] * 9
        lib.kda_chunk_fwd_host_buffer_size.restype = szt
        lib.kda_chunk_fwd_host.argtypes = [vp] * 9 + [i32] * 7 + [i32, i32, vp, szt, vp, vp, vp]
        lib.kda_chunk_fwd_host.restype = i32
        lib.kda_chunk_fwd_noalloc.argtypes = [vp] * 9 + [i32] * 7 + [i32, vp]
        lib.kda_chunk_fwd_noalloc.restype = i32
        lib.kda_chunk_bwd_workspace_size.argtypes = [i32] * 6
        lib.kda_chunk_bwd_workspace_size.restype = szt
        lib.kda_chunk_bwd.argtypes = [vp] * 15 + [i32] * 6 + [i32, vp, szt, vp]
        lib.kda_chunk_bwd.restype = i32
        lib.kda_gdn_chunk_bwd.argtypes = lib.kda_chunk_bwd.argtypes
        lib.kda_gdn_chunk_bwd.restype = i32
        lib.kda_chunk_bwd_prep_workspace_size.argtypes = [i32] * 6
        lib.kda_chunk_bwd_prep_workspace_size.restype = szt
        lib.kda_chunk_bwd_prep.argtypes = [vp] * 4 + [i32] + [vp] * 11 + [i32] * 6 + [i32, vp, szt, vp]
        lib.kda_chunk_bwd_prep.restype = i32
        lib.kda_set_segment_chunks.argtypes = [i32]
        lib.kda_set_segment_chunks.restype = i32
        lib.kda_segment_chunks.argtypes = [i32] * 4
        lib.kda_segment_chunks.restype = i32
        lib.kda_set_local_kernel.argtypes = [i32]
        lib.kda_set_local_kernel.restype = i32
        lib.kda_set_prefill_path.argtypes = [i32]
        lib.kda_set_prefill_path.restype = i32
        lib.kda_chunk_fwd_phases.argtypes = [i32] * 8
        lib.kda_chunk_fwd_phases.restype = i32
        lib.kda_selftest_bounded_wait.argtypes = [ctypes.c_ulonglong, vp]
        lib.kda_selftest_bounded_wait.restype = i32
        lib.kda_version.argtypes = []
        lib.kda_version.restype = i32
        _lib = lib
        return lib


def _check(st):
    if st != KDA_OK:
        raise KDAError(st, load_library().kda_last_error().decode())


def last_error() -> str:
    return load_library().kda_last_error().decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return KDA_BF16
    if t.dtype == torch.float32:
        return KDA_F32
    raise TypeError(f"q/k/v must be bfloat16 or float32, got {t.dtype}")


def _need_cuda(*ts):
    dev = None
    for t in ts:
        if t is not None:
            if not t.is_cuda:
                raise ValueError("tensors must be on a CUDA device (use chunk_fwd_host for host buffers)")
            if not t.is_contiguous():
                raise ValueError("tensors must be contiguous")
            if dev is None:
                dev = t.device
            elif t.device != dev:
                raise ValueError(f"tensors on different devices ({dev} and {t.device})")


def _prefill_shapes(fn, q, k, v, g, beta, S0, cu_seqlens, o=None, S_out=None):
    """Checks every prefill argument's dtype and shape against q's [B,T,H,dk]
    and v's dv (the C ABI sees only pointers and sizes, so a wrong dtype or
    shape here would be read past its end on the device), then that all are
    contiguous CUDA tensors on one device.  Returns (B, T, H, dk, dv,
    num_seqs, N)."""
    if q.dim() != 4 or k.shape != q.shape or v.dim() != 4 or v.shape[:3] != q.shape[:3]:
        raise ValueError(f"q, k must be [B,T,H,dk] and v [B,T,H,dv], got {tuple(q.shape)}, {tuple(k.shape)}, "
                         f"{tuple(v.shape)}")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError(f"q, k, v must share one dtype, got {q.dtype}, {k.dtype}, {v.dtype}")
    _dtype_code(q)
    prep = fn == "kda_chunk_fwd_prep"
    if g.dtype not in ((torch.float32, torch.bfloat16) if prep else (torch.float32,)) or beta.dtype != torch.float32:
        raise TypeError("g (a) and beta (b) must be float32 (a may be bfloat16)")
    g_shape = (B, T, H) if fn == "kda_gdn_chunk_fwd" else (B, T, H, dk)
    if tuple(g.shape) != g_shape or tuple(beta.shape) != (B, T, H):
        raise ValueError(f"g must be {g_shape} and beta {(B, T, H)}, got {tuple(g.shape)}, {tuple(beta.shape)}")
    if cu_seqlens is not None:
        if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2:
            raise TypeError("cu_seqlens must be a 1-D int32 tensor of num_seqs + 1 entries")
        if B != 1:
            raise ValueError("packed sequences (cu_seqlens) need B == 1")
    num_seqs = 0 if cu_seqlens is None else cu_seqlens.numel() - 1
    N = num_seqs if cu_seqlens is not None else B
    for name, t in (("S0", S0), ("S_out", S_out)):
        if t is not None and (t.dtype != torch.float32 or tuple(t.shape) != (N, H, dk, dv)):
            raise ValueError(f"{name} must be float32 {(N, H, dk, dv)}, got {t.dtype} {tuple(t.shape)}")
    if o is not None and (o.dtype != q.dtype or tuple(o.shape) != (B, T, H, dv)):
        raise ValueError(f"o must be {q.dtype} {(B, T, H, dv)}, got {o.dtype} {tuple(o.shape)}")
    _need_cuda(q, k, v, g, beta, S0, cu_seqlens, o, S_out)
    return B, T, H, dk, dv, num_seqs, N


def workspace_size(B, T, H, dk, dv, num_seqs=0, chunk_size=64, dtype=torch.bfloat16) -> int:
    code = KDA_BF16 if dtype == torch.bfloat16 else KDA_F32
    return int(load_library().kda_chunk_fwd_workspace_size(B, T, H, dk, dv, num_seqs, chunk_size, code))


def chunk_fwd(q, k, v, g, beta, S0=None, cu_seqlens=None, chunk_size=64, output_final_state=True,
              o=None, S_out=None, workspace=None):
    """Chunkwise KDA prefill.  q, k, g: [B,T,H,dk]; v: [B,T,H,dv]; beta: [B,T,H];
    S0: [N,H,dk,dv] fp32 or None; cu_seqlens: int32 [N+1] (B == 1) or None.
    Returns (o, S_out) with S_out None when output_final_state is False."""
    return _chunk_fwd("kda_chunk_fwd", q, k, v, g, beta, S0, cu_seqlens, chunk_size, output_final_state,
                      o, S_out, workspace)


def gdn_chunk_fwd(q, k, v, g, beta, S0=None, cu_seqlens=None, chunk_size=64, output_final_state=True,
                  o=None, S_out=None, workspace=None):
    """Gated DeltaNet prefill: as chunk_fwd with one gate per token and head,
    g: [B,T,H] fp32 (log alpha)."""
    return _chunk_fwd("kda_gdn_chunk_fwd", q, k, v, g, beta, S0, cu_seqlens, chunk_size,
                      output_final_state, o, S_out, workspace)


def chunk_fwd_prep(q, k, v, a, b, S0=None, cu_seqlens=None, chunk_size=64, output_final_state=True,
                   o=None, S_out=None, workspace=None):
    """KDA prefill from raw projections: q, k [B,T,H,dk] unnormalised; a [B,T,H,dk]
    raw gate logits (bf16 or fp32; log alpha = -softplus(a)); b [B,T,H] fp32 raw
    beta logits (beta = sigmoid(b)).  q and k are L2-normalised per (token, head)
    inside the kernels."""
    return _chunk_fwd("kda_chunk_fwd_prep", q, k, v, a, b, S0, cu_seqlens, chunk_size, output_final_state,
                      o, S_out, workspace)


def _chunk_fwd(fn, q, k, v, g, beta, S0, cu_seqlens, chunk_size, output_final_state, o, S_out,
               workspace):
    lib = load_library()
    B, T, H, dk, dv, num_seqs, N = _prefill_shapes(fn, q, k, v, g, beta, S0, cu_seqlens, o, S_out)
    _need_cuda(workspace, q)
    prep = fn == "kda_chunk_fwd_prep"
    with torch.cuda.device(q.device):
        if o is None:
            o = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
        if S_out is None and output_final_state:
            S_out = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
        ws_need = workspace_size(B, T, H, dk, dv, num_seqs, chunk_size, q.dtype)
        if workspace is None and ws_need:
            workspace = torch.empty(ws_need, dtype=torch.uint8, device=q.device)
        ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
        gargs = (_ptr(g), _dtype_code(g)) if prep else (_ptr(g),)
        st = getattr(lib, fn)(_ptr(q), _ptr(k), _ptr(v), *gargs, _ptr(beta), _ptr(S0), _ptr(o),
                              _ptr(S_out), _ptr(cu_seqlens), num_seqs, B, T, H, dk, dv, chunk_size,
                              _dtype_code(q), _ptr(workspace), ws_bytes, _stream_handle(q.device))
    _check(st)
    return o, S_out


def chunk_fwd_noalloc(q, k, v, g, beta, S0=None, cu_seqlens=None, chunk_size=64, o=None, S_out=None):
    """chunk_fwd through kda_chunk_fwd_noalloc: no workspace is passed or
    allocated (the library's built-in scratch array is used; o and S_out are
    allocated here only when not given).  The arguments are checked exactly as
    chunk_fwd checks them, and the call runs with q's device current (the
    library looks up the built-in array of the current device).  Returns
    (o, S_out)."""
    lib = load_library()
    B, T, H, dk, dv, num_seqs, N = _prefill_shapes("kda_chunk_fwd", q, k, v, g, beta, S0, cu_seqlens, o, S_out)
    with torch.cuda.device(q.device):
        if o is None:
            o = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
        if S_out is None:
            S_out = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
        st = lib.kda_chunk_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0), _ptr(o),
                                       _ptr(S_out), _ptr(cu_seqlens), num_seqs, B, T, H, dk, dv, chunk_size,
                                       _dtype_code(q), _stream_handle(q.device))
    _check(st)
    return o, S_out


def recurrent_step(q, k, v, g, beta, S, o=None):
    """One decode token per sequence: q, k, g [N,H,dk]; v [N,H,dv]; beta [N,H];
    S [N,H,dk,dv] fp32 updated in place.  Returns o [N,H,dv]."""
    return _recurrent_step("kda_recurrent_step", q, k, v, g, beta, S, o)


def gdn_recurrent_step(q, k, v, g, beta, S, o=None):
    """Gated DeltaNet decode step: as recurrent_step with g [N,H] fp32."""
    return _recurrent_step("kda_gdn_recurrent_step", q, k, v, g, beta, S, o)


def recurrent_step_prep(q, k, v, a, b, S, o=None):
    """Decode step from raw projections (see chunk_fwd_prep): a [N,H,dk] bf16 or
    fp32 raw gate logits, b [N,H] fp32 raw beta logits."""
    return _recurrent_step("kda_recurrent_step_prep", q, k, v, a, b, S, o)


def chunk_bwd(q, k, v, g, beta, dout, S0=None, dS_T=None, cu_seqlens=None, workspace=None,
              need_dS0=True):
    """Backward pass of chunk_fwd: gradients of a loss L with respect to q, k,
    v, g, beta (and S0) given dout = dL/do and dS_T = dL/dS_final (or None).
    Returns a dict of fp32 tensors dq, dk, dv, dg [B,T,H,d], dbeta [B,T,H] and
    dS0 [N,H,dk,dv] (None when need_dS0 is False)."""
    return _chunk_bwd("kda_chunk_bwd", q, k, v, g, beta, dout, S0, dS_T, cu_seqlens, workspace, need_dS0)


def gdn_chunk_bwd(q, k, v, g, beta, dout, S0=None, dS_T=None, cu_seqlens=None, workspace=None,
                  need_dS0=True):
    """Backward pass of gdn_chunk_fwd (one gate per token and head): as
    chunk_bwd with g [B,T,H] fp32, and dg [B,T,H]."""
    return _chunk_bwd("kda_gdn_chunk_bwd", q, k, v, g, beta, dout, S0, dS_T, cu_seqlens, workspace, need_dS0)


def chunk_bwd_prep(q, k, v, a, b, dout, S0=None, dS_T=None, cu_seqlens=None, workspace=None, need_dS0=True):
    """Backward pass of chunk_fwd_prep (raw projections): gradients of a loss L
    with respect to the RAW q, k [B,T,H,dk], v, the gate logits a [B,T,H,dk]
    (bf16 or fp32) and the beta logits b [B,T,H] fp32 (and S0), given dout =
    dL/do and dS_T = dL/dS_final (or None).  Returns a dict of fp32 tensors dq,
    dk, dv, da, db and dS0 (None when need_dS0 is False)."""
    lib = load_library()
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    num_seqs = 0 if cu_seqlens is None else cu_seqlens.numel() - 1
    N = num_seqs if cu_seqlens is not None else B
    if a.dtype not in (torch.float32, torch.bfloat16) or b.dtype != torch.float32 or dout.dtype != q.dtype:
        raise TypeError("a must be float32 or bfloat16, b float32, and dout must have q's dtype")
    if tuple(a.shape) != (B, T, H, dk) or tuple(b.shape) != (B, T, H) or tuple(dout.shape) != (B, T, H, dv):
        raise ValueError("a must be [B,T,H,dk], b [B,T,H], dout [B,T,H,dv]")
    _need_cuda(q, k, v, a, b, dout, S0, dS_T, cu_seqlens, workspace)
    f32 = dict(dtype=torch.float32, device=q.device)
    with torch.cuda.device(q.device):
        out = dict(dq=torch.empty((B, T, H, dk), **f32), dk=torch.empty((B, T, H, dk), **f32),
                   dv=torch.empty((B, T, H, dv), **f32), da=torch.empty((B, T, H, dk), **f32),
                   db=torch.empty((B, T, H), **f32),
                   dS0=torch.empty((N, H, dk, dv), **f32) if need_dS0 else None)
        need = int(lib.kda_chunk_bwd_prep_workspace_size(B, T, H, dk, dv, num_seqs))
        if workspace is None and need:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
        st = lib.kda_chunk_bwd_prep(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _dtype_code(a), _ptr(b), _ptr(S0),
                                    _ptr(dout), _ptr(dS_T), _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]),
                                    _ptr(out["da"]), _ptr(out["db"]), _ptr(out["dS0"]), _ptr(cu_seqlens), num_seqs,
                                    B, T, H, dk, dv, _dtype_code(q), _ptr(workspace), ws_bytes,
                                    _stream_handle(q.device))
    _check(st)
    return out


def _chunk_bwd(fn, q, k, v, g, beta, dout, S0, dS_T, cu_seqlens, workspace, need_dS0):
    lib = load_library()
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    num_seqs = 0 if cu_seqlens is None else cu_seqlens.numel() - 1
    N = num_seqs if cu_seqlens is not None else B
    if g.dtype != torch.float32 or beta.dtype != torch.float32 or dout.dtype != q.dtype:
        raise TypeError("g and beta must be float32 and dout must have q's dtype")
    g_shape = (B, T, H) if fn == "kda_gdn_chunk_bwd" else (B, T, H, dk)
    if tuple(g.shape) != g_shape or tuple(beta.shape) != (B, T, H) or tuple(dout.shape) != (B, T, H, dv):
        raise ValueError(f"g must be {list(g_shape)}, beta [B,T,H], dout [B,T,H,dv]")
    _need_cuda(q, k, v, g, beta, dout, S0, dS_T, cu_seqlens, workspace)
    f32 = dict(dtype=torch.float32, device=q.device)
    with torch.cuda.device(q.device):
        out = dict(dq=torch.empty((B, T, H, dk), **f32), dk=torch.empty((B, T, H, dk), **f32),
                   dv=torch.empty((B, T, H, dv), **f32), dg=torch.empty(g_shape, **f32),
                   dbeta=torch.empty((B, T, H), **f32),
                   dS0=torch.empty((N, H, dk, dv), **f32) if need_dS0 else None)
        need = int(lib.kda_chunk_bwd_workspace_size(B, T, H, dk, dv, num_seqs))
        if workspace is None and need:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
        st = getattr(lib, fn)(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0), _ptr(dout), _ptr(dS_T),
                              _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dg"]),
                              _ptr(out["dbeta"]), _ptr(out["dS0"]), _ptr(cu_seqlens), num_seqs, B, T, H, dk, dv,
                              _dtype_code(q), _ptr(workspace), ws_bytes, _stream_handle(q.device))
    _check(st)
    return out


def _recurrent_step(fn, q, k, v, g, beta, S, o):
    lib = load_library()
    _need_cuda(q, k, v, g, beta, S, o)
    N, H, dk = q.shape
    dv = v.shape[-1]
    prep = fn == "kda_recurrent_step_prep"
    g_ok = g.dtype in ((torch.float32, torch.bfloat16) if prep else (torch.float32,))
    if S.dtype != torch.float32 or not g_ok or beta.dtype != torch.float32:
        raise TypeError("S, g (a) and beta (b) must be float32 (a may be bfloat16)")
    g_shape = (N, H) if fn == "kda_gdn_recurrent_step" else (N, H, dk)
    if tuple(g.shape) != g_shape or tuple(beta.shape) != (N, H) or tuple(S.shape) != (N, H, dk, dv):
        raise ValueError(f"g must be {g_shape}, beta {(N, H)}, S {(N, H, dk, dv)}")
    if o is None:
        o = torch.empty((N, H, dv), dtype=q.dtype, device=q.device)
    gargs = (_ptr(g), _dtype_code(g)) if prep else (_ptr(g),)
    st = getattr(lib, fn)(_ptr(q), _ptr(k), _ptr(v), *gargs, _ptr(beta), _ptr(S), _ptr(o),
                          N, H, dk, dv, _dtype_code(q), _stream_handle(q.device))
    _check(st)
    return o


class HostPrefill:
    """chunk_fwd over HOST tensors through the C ABI's kda_chunk_fwd_host: the
    library copies the inputs to the device, runs the prefill and copies o and
    S_out back into host buffers, pipelined over `pieces` groups of batch rows
    on three streams (host->device copies, the prefill on the current stream,
    device->host copies).  This class only keeps the device buffer the library
    asks for, the two copy streams and the pinned output buffers; the current
    stream waits for the last copy back, so synchronising it covers the call.
    Host inputs should be pinned (page-locked) for the copies to overlap."""

    def __init__(self, like: dict, device="cuda", chunk_size=64, pieces=None):
        self.device = torch.device(device)
        self.chunk_size = chunk_size
        q, v = like["q"], like["v"]
        B, T, H, dk = q.shape
        cu = like.get("cu_seqlens")
        self.num_seqs = 0 if cu is None else cu.numel() - 1
        N = self.num_seqs if cu is not None else B
        self.shape = (B, T, H, dk, v.shape[-1])
        self.dtype = q.dtype
        self.pieces = max(1, min(B, pieces if pieces else 8))
        self.o_host = torch.empty((B, T, H, v.shape[-1]), dtype=q.dtype, pin_memory=True)
        self.S_host = torch.empty((N, H, dk, v.shape[-1]), dtype=torch.float32, pin_memory=True)
        lib = load_library()
        nbytes = int(lib.kda_chunk_fwd_host_buffer_size(B, T, H, dk, v.shape[-1], self.num_seqs, chunk_size,
                                                         _dtype_code(q), self.pieces))
        self.buf = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=self.device)
        self.buf_bytes = nbytes
        self.s_in = torch.cuda.Stream(self.device)
        self.s_out = torch.cuda.Stream(self.device)

    def h2d_bytes(self, host: dict) -> int:
        names = ("q", "k", "v", "g", "beta", "S0", "cu_seqlens")
        return int(sum(t.numel() * t.element_size() for n, t in host.items() if t is not None and n in names))

    def d2h_bytes(self) -> int:
        return int(self.o_host.numel() * self.o_host.element_size() + self.S_host.numel() * 4)

    def __call__(self, host: dict):
        lib = load_library()
        B, T, H, dk, dv = self.shape
        for n in ("q", "k", "v", "g", "beta", "S0", "cu_seqlens"):
            t = host.get(n)
            if t is not None and (t.is_cuda or not t.is_contiguous()):
                raise ValueError(f"{n} must be a contiguous host tensor")
        with torch.cuda.device(self.device):
            st = lib.kda_chunk_fwd_host(
                _ptr(host["q"]), _ptr(host["k"]), _ptr(host["v"]), _ptr(host["g"]), _ptr(host["beta"]),
                _ptr(host.get("S0")), _ptr(self.o_host), _ptr(self.S_host), _ptr(host.get("cu_seqlens")),
                self.num_seqs, B, T, H, dk, dv, self.chunk_size, _dtype_code(host["q"]), self.pieces,
                _ptr(self.buf), self.buf_bytes, _stream_handle(self.device),
                ctypes.c_void_p(self.s_in.cuda_stream), ctypes.c_void_p(self.s_out.cuda_stream))
        _check(st)
        return self.o_host, self.S_host


def chunk_fwd_host(host: dict, chunk_size=64, device="cuda"):
    """One-shot host-buffer prefill (see HostPrefill); synchronises before returning."""
    runner = HostPrefill(host, device, chunk_size)
    o, S = runner(host)
    torch.cuda.current_stream(runner.device).synchronize()
    return o, S


def device_error(device=None) -> int:
    """Read-and-clear the device error word set by bounded waits (synchronises)."""
    lib = load_library()
    code = ctypes.c_int(0)
    _check(lib.kda_device_error(ctypes.byref(code), _stream_handle(device)))
    return code.value


def set_segment_chunks(chunks: int) -> None:
    """Sequence segments of the tensor-core prefill for this thread's later
    calls: 0 = automatic (default), L > 0 = L chunks per segment, < 0 = off."""
    _check(load_library().kda_set_segment_chunks(int(chunks)))


def set_local_kernel(variant: int) -> None:
    """Chunk-local kernel of the tensor-core prefill for this thread's later
    calls: 0 = the warp-specialised kernel where it applies (default),
    1 = the two-CTA-per-SM kernel always."""
    _check(load_library().kda_set_local_kernel(int(variant)))
    _tls.local_kernel = int(variant)


def set_prefill_path(path: int) -> None:
    """Tensor-core prefill for this thread's later calls: 0 = automatic
    (default: the single pass when the (sequence, head) units fill their waves
    of one unit per SM to 80%, or for packed sequences with a unit per SM; the
    two-kernel path otherwise), 1 = the single-pass kernel, 2 = the two-kernel
    path."""
    _check(load_library().kda_set_prefill_path(int(path)))
    _tls.prefill_path = int(path)


def prefill_phases(B, T, H, num_seqs=0, dk=128, dv=128, chunk_size=64, dtype=torch.bfloat16) -> int:
    """Phases of one chunk_fwd call with these sizes on the current device and
    this thread's settings (1: the fp32 path, or the single pass: its set-up
    kernel and its plain and precise instances; 2: the two-kernel path's
    chunk-local phase, then its state pass with the precise fallback)."""
    code = KDA_BF16 if dtype == torch.bfloat16 else KDA_F32
    return int(load_library().kda_chunk_fwd_phases(B, T, H, num_seqs, dk, dv, chunk_size, code))


def uses_fused_kernel(B, T, H, num_seqs=0, dk=128, dv=128, chunk_size=64, dtype=torch.bfloat16) -> bool:
    """Whether a prefill call of these sizes on this thread runs the
    single-pass kernel."""
    return (launches_per_chunk_fwd(dk, dv, chunk_size, dtype) == 2
            and prefill_phases(B, T, H, num_seqs, dk, dv, chunk_size, dtype) == 1)


def uses_ws_kernel(gate="log_channel", packed=False, dk=128, dv=128, chunk_size=64, dtype=torch.bfloat16) -> bool:
    """Whether a prefill call of this kind on this thread runs the
    warp-specialised chunk-local kernel: tensor-core path, any layout (packed
    sequences first build a chunk table), any gate ("log_channel" = KDA,
    "log_token" = Gated DeltaNet, "logit" = raw gate logits with the
    preparation fused)."""
    if gate not in ("log_channel", "log_token", "logit"):
        raise ValueError(f"gate {gate!r}")
    return launches_per_chunk_fwd(dk, dv, chunk_size, dtype) == 2 and getattr(_tls, "local_kernel", 0) == 0


def segment_chunks(B, T, H, num_seqs=0) -> int:
    """Chunks per segment the prefill would use for these sizes (0 = none)."""
    return int(load_library().kda_segment_chunks(B, T, H, num_seqs))


def selftest_bounded_wait(limit_ns=50_000_000, device=None):
    """Run the library's bounded-wait self-check on the current stream: a wait
    that nothing completes gives up after limit_ns and sets the device error
    word (read it with device_error())."""
    dev = torch.device("cuda") if device is None else torch.device(device)
    _check(load_library().kda_selftest_bounded_wait(int(limit_ns), _stream_handle(dev)))


def launches_per_chunk_fwd(dk, dv, chunk_size, dtype=torch.bfloat16) -> int:
    code = KDA_BF16 if dtype == torch.bfloat16 else KDA_F32
    return int(load_library().kda_chunk_fwd_launches(dk, dv, chunk_size, code))


def kernel_names(dk, dv, chunk_size, dtype=torch.bfloat16, gate="log_channel", packed=False, shape=None):
    """Phases of one chunk_fwd call, named by the kernel that does each one's
    work.  ``shape`` = (B, T, H, num_seqs) selects the path those sizes take
    (single pass or two kernels); without it the two-kernel names are given
    (the chunk-local phase of the warp-specialised path also launches the
    two-CTA kernel over the chunks it passed on, usually none)."""
    n = launches_per_chunk_fwd(dk, dv, chunk_size, dtype)
    if n == 1:
        return KERNELS_SIMT
    if shape is not None and uses_fused_kernel(*shape, dk=dk, dv=dv, chunk_size=chunk_size, dtype=dtype):
        return (KERNEL_FUSED,)
    first = KERNEL_WS if uses_ws_kernel(gate, packed, dk, dv, chunk_size, dtype) else KERNELS_TC[0]
    return (first,) + KERNELS_TC[1:n]


def chunk_fwd_kernel_sequence(B, T, H, dk=128, dv=128, chunk_size=64, dtype=torch.bfloat16, gate="log_channel",
                              num_seqs=0):
    """Every kernel one chunk_fwd call launches, in order."""
    if launches_per_chunk_fwd(dk, dv, chunk_size, dtype) == 1:
        return list(KERNELS_SIMT)
    if uses_fused_kernel(B, T, H, num_seqs, dk, dv, chunk_size, dtype):
        # the plain instance, then the precise one (it returns at once unless the
        # plain one marked a unit with near-parallel keys)
        return ["kda_fused_setup_kernel", KERNEL_FUSED, KERNEL_FUSED]
    # the precise fallback's set-up first and its single-pass kernel last (it
    # returns at once unless a chunk-local kernel met near-parallel keys)
    seq = ["kda_fused_setup_kernel"] + (["kda_ws_chunk_table_kernel"] if num_seqs > 0 else [])
    if uses_ws_kernel(gate, num_seqs > 0, dk, dv, chunk_size, dtype):
        seq += [KERNEL_WS, KERNELS_TC[0]]
    else:
        seq += [KERNELS_TC[0]]
    if segment_chunks(B, T, H, num_seqs) > 0:
        return seq + [KERNELS_TC[1], "kda_tc_seg_combine_kernel", KERNELS_TC[1], KERNEL_FUSED]
    return seq + [KERNELS_TC[1], KERNEL_FUSED]


def profile_chunk_fwd(call, stream, repeats=3, dk=128, dv=128, chunk_size=64, dtype=torch.bfloat16,
                      gate="log_channel", packed=False, shape=None):
    """Run ``call()`` (one chunk_fwd call) ``repeats`` times with the library's
    event hook set and return {phase's kernel name: mean ms per call}.
    ``shape`` = (B, T, H, num_seqs) of the call (selects its path)."""
    lib = load_library()
    names = kernel_names(dk, dv, chunk_size, dtype, gate, packed, shape)
    n = len(names)
    events = [torch.cuda.Event(enable_timing=True) for _ in range((n + 1) * repeats)]
    for e in events:  # torch creates the underlying event lazily, at its first record
        e.record(stream)
    totals = [0.0] * n
    for r in range(repeats):
        evs = events[r * (n + 1):(r + 1) * (n + 1)]
        arr = (ctypes.c_void_p * (n + 1))(*[ctypes.c_void_p(e.cuda_event) for e in evs])
        _check(lib.kda_profile_events(arr, n + 1))
        try:
            call()
        finally:
            lib.kda_profile_events(None, 0)
        evs[-1].synchronize()
        for i in range(n):
            totals[i] += evs[i].elapsed_time(evs[i + 1])
    return {name: t / repeats for name, t in zip(names, totals)}


# Algorithmic bytes per launch, per kernel, for dk = dv = 128 (see the design
# notes): the prefill's minimum traffic is q, k, v (bf16), g (fp32), beta, o
# (bf16) = 1540 B per token-head plus the fp32 initial/final state per unit.
# In the two-kernel tensor-core path the chunk-local kernel also writes, and
# the state pass reads, the per-chunk WY image (1160 B per token-head).
TC_IMAGE_BYTES_PER_TOKEN_HEAD = 1160


def algorithmic_bytes_per_launch(kernel, token_heads, units, d=128, with_state_in=False,
                                 gate_per_channel=True, gate_bytes=4):
    """Bytes one launch must move.  The gate has d values per token-head (KDA)
    or one (Gated DeltaNet, gate_per_channel=False), of gate_bytes each (4 for
    fp32 log alpha or logits, 2 for bf16 logits)."""
    state = d * d * 4 * units
    gate = gate_bytes * d if gate_per_channel else gate_bytes
    if kernel == "kda_chunk_simt_kernel":
        return token_heads * (3 * 2 * d + gate + 4 + 2 * d) + state * (2 if with_state_in else 1)
    if kernel == KERNEL_FUSED:
        return token_heads * (3 * 2 * d + gate + 4 + 2 * d) + state * (2 if with_state_in else 1)
    if kernel in ("kda_tc_chunk_local_kernel", KERNEL_WS):
        return token_heads * (3 * 2 * d + gate + 4 + TC_IMAGE_BYTES_PER_TOKEN_HEAD)
    if kernel == "kda_tc_state_pass_kernel":
        return token_heads * (TC_IMAGE_BYTES_PER_TOKEN_HEAD + 2 * d) + state * (2 if with_state_in else 1)
    raise KeyError(kernel)


def version() -> int:
    return int(load_library().kda_version())


__all__ = ["chunk_fwd", "chunk_fwd_noalloc", "recurrent_step", "chunk_fwd_host", "HostPrefill", "workspace_size",
           "launches_per_chunk_fwd", "kernel_names", "profile_chunk_fwd", "algorithmic_bytes_per_launch",
           "set_local_kernel", "uses_ws_kernel", "chunk_fwd_kernel_sequence", "set_prefill_path",
           "prefill_phases", "uses_fused_kernel",
           "last_error", "device_error", "version", "load_library", "lib_path", "KDAError", "EXPORTED"]
