"""Plain fp64 CPU oracle for the Kimi Delta Attention (KDA) recurrence.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product path
(``kimi_delta_attention_31_b200``) never imports it, and the two share no code.

The arithmetic lives in ``kda_oracle.c`` (plain C99, fp64, OpenMP over
independent (sequence, head) units); this module only builds it with gcc and
marshals numpy arrays through ctypes.

Functions
---------
recurrent(...)  token-by-token definition ("Kimi K3 notes 1: KDA" section 4/5;
                "Deriving KDA from scratch" sections 3-5).
chunk(...)      chunkwise schedule in fp64 with pairwise exponentials and plain
                forward substitution ("Deriving KDA from scratch" section 6;
                "Linear / sparse attention" tutorial section 6.2).
gdn_recurrent(...)  Gated DeltaNet (one gate per token and head): the
                recurrence above with the gate broadcast over key channels.
prep(...)       input preparation from raw projections (q, k L2-normalised,
                log alpha = -softplus(a), beta = sigmoid(b)); recurrent_prep
                chains it with recurrent().

Inputs are widened exactly to fp64 (bf16 and fp32 values are representable),
so the rounding of the inputs the GPU sees is not counted as error.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB = os.path.join(_HERE, "libkda_oracle.so")
_lock = threading.Lock()
_lib = None

NO_ERASE = 0x1
# Planted mistakes for the mutation tests (tests/test_oracle_mutations.py).
MUT_GATE_ON_VALUE_AXIS = 0x100
MUT_PREDICT_UNDECAYED = 0x200
MUT_OUTPUT_PRE_WRITE = 0x400
MUT_NO_DECAY = 0x800
MUT_READ_TRANSPOSED = 0x1000
MUT_ERROR_SIGN = 0x2000


def build(force: bool = False) -> str:
    """Compile kda_oracle.c into libkda_oracle.so with gcc (-O2 -fopenmp)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            dp = ctypes.POINTER(ctypes.c_double)
            ip = ctypes.POINTER(ctypes.c_int64)
            common = [dp, dp, dp, dp, dp, dp, dp, dp, ip, ctypes.c_int, ctypes.c_int,
                      ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int]
            lib.kda_oracle_recurrent.argtypes = common + [ctypes.c_int, dp, ctypes.c_int]
            lib.kda_oracle_recurrent.restype = ctypes.c_int
            lib.kda_oracle_chunk.argtypes = common + [ctypes.c_int, ctypes.c_int]
            lib.kda_oracle_chunk.restype = ctypes.c_int
            lib.kda_oracle_max_threads.argtypes = []
            lib.kda_oracle_max_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor: widen exactly on the host
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a, typ=ctypes.c_double):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(typ))


def _shapes(q, v, cu_seqlens):
    if q.ndim != 4 or v.ndim != 4:
        raise ValueError("q/k/g must be [B,T,H,dk] and v [B,T,H,dv]")
    B, T, H, dk = q.shape
    dv = v.shape[3]
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
        if B != 1:
            raise ValueError("packed (cu_seqlens) inputs need B == 1")
        N = cu.shape[0] - 1
    else:
        cu = None
        N = B
    return B, T, H, dk, dv, N, cu


def max_threads() -> int:
    return int(_load().kda_oracle_max_threads())


def recurrent(q, k, v, g, beta, S0=None, cu_seqlens=None, flags=0, return_history=False,
              num_threads=0):
    """Token-by-token fp64 KDA.  Returns (o, S_out[, S_hist]) as float64 arrays.

    q, k, g: [B,T,H,dk]; v: [B,T,H,dv]; beta: [B,T,H]; S0: [N,H,dk,dv] or None.
    """
    lib = _load()
    q, k, v, g, beta, S0 = (_f64(x) for x in (q, k, v, g, beta, S0))
    B, T, H, dk, dv, N, cu = _shapes(q, v, cu_seqlens)
    o = np.zeros((B, T, H, dv), np.float64)
    S_out = np.zeros((N, H, dk, dv), np.float64)
    hist = np.zeros((B, T, H, dk, dv), np.float64) if return_history else None
    rc = lib.kda_oracle_recurrent(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0), _ptr(o), _ptr(S_out),
        _ptr(cu, ctypes.c_int64), N if cu is not None else 0, B, T, H, dk, dv,
        int(flags), _ptr(hist), int(num_threads))
    if rc != 0:
        raise ValueError(f"kda_oracle_recurrent failed with code {rc}")
    return (o, S_out, hist) if return_history else (o, S_out)


def gdn_recurrent(q, k, v, g, beta, S0=None, cu_seqlens=None, num_threads=0):
    """Gated DeltaNet, token by token in fp64: one decay per token and head
    ("Kimi K3 notes 1: KDA" section 3; "Linear / sparse attention" tutorial
    section 5.2), g: [B,T,H].  KDA with every key channel's gate equal to it,
    so the per-channel recurrence runs on g broadcast over dk (the oracle's
    pin 6 checks that reduction against the tutorial's own Gated DeltaNet
    update).  Returns (o, S_out)."""
    g = _f64(g)
    dk = (q.shape[-1])
    if g.ndim != 3:
        raise ValueError("Gated DeltaNet g must be [B,T,H]")
    g_full = np.ascontiguousarray(np.broadcast_to(g[..., None], g.shape + (dk,)))
    return recurrent(q, k, v, g_full, beta, S0, cu_seqlens, num_threads=num_threads)


def prep(q, k, a, b):
    """Input preparation in fp64, from raw projections ("Kimi K3 notes 1: KDA"
    section 4: q and k are L2-normalised; "Linear / sparse attention" tutorial
    section 10: beta and the decay come from bounded activations).  Per token
    and head:
        q / max(|q|_2, 1e-12),  k / max(|k|_2, 1e-12)   (over the last axis)
        g = log alpha = -softplus(a) = -log(1 + e^a)
        beta = sigmoid(b) = 1 / (1 + e^-b)
    Returns (q, k, g, beta) as float64 arrays."""
    q, k, a, b = (_f64(x) for x in (q, k, a, b))
    q = q / np.maximum(np.linalg.norm(q, axis=-1, keepdims=True), 1e-12)
    k = k / np.maximum(np.linalg.norm(k, axis=-1, keepdims=True), 1e-12)
    g = -np.logaddexp(0.0, a)          # log(e^0 + e^a)
    beta = 0.5 * (1.0 + np.tanh(0.5 * b))  # = 1 / (1 + e^-b), without overflow
    return q, k, g, beta


def recurrent_prep(q, k, v, a, b, S0=None, cu_seqlens=None, num_threads=0):
    """prep() followed by the token-by-token recurrence.  Returns (o, S_out)."""
    qn, kn, g, beta = prep(q, k, a, b)
    return recurrent(qn, kn, v, g, beta, S0, cu_seqlens, num_threads=num_threads)


def chunk(q, k, v, g, beta, S0=None, cu_seqlens=None, chunk_size=16, num_threads=0):
    """Chunkwise fp64 KDA (pairwise exps, forward substitution).  Returns (o, S_out)."""
    lib = _load()
    q, k, v, g, beta, S0 = (_f64(x) for x in (q, k, v, g, beta, S0))
    B, T, H, dk, dv, N, cu = _shapes(q, v, cu_seqlens)
    o = np.zeros((B, T, H, dv), np.float64)
    S_out = np.zeros((N, H, dk, dv), np.float64)
    rc = lib.kda_oracle_chunk(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0), _ptr(o), _ptr(S_out),
        _ptr(cu, ctypes.c_int64), N if cu is not None else 0, B, T, H, dk, dv,
        int(chunk_size), int(num_threads))
    if rc != 0:
        raise ValueError(f"kda_oracle_chunk failed with code {rc}")
    return o, S_out


def rel_rms_per_slice(x, ref, axis_unit=(0, 2)):
    """max over (sequence, head) slices of ||x - ref||_2 / ||ref||_2.

    ``x`` and ``ref`` are [B,T,H,d] (outputs) or [N,H,dk,dv] (states); the slice
    is one (sequence, head) pair.  Where ||ref|| < 1e-30 the absolute RMS is
    used instead.  This is the tolerance metric the parity tests apply.
    """
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    if x.shape != ref.shape:
        raise ValueError(f"shape mismatch {x.shape} vs {ref.shape}")
    if x.ndim == 4 and axis_unit == (0, 2):  # [B,T,H,d]: slice = (b, h) over (T, d)
        d = (x - ref)
        num = np.sqrt((d * d).sum(axis=(1, 3)))
        den = np.sqrt((ref * ref).sum(axis=(1, 3)))
        cnt = x.shape[1] * x.shape[3]
    else:  # states [N,H,dk,dv]: slice = (n, h)
        d = (x - ref)
        num = np.sqrt((d * d).sum(axis=(2, 3)))
        den = np.sqrt((ref * ref).sum(axis=(2, 3)))
        cnt = x.shape[2] * x.shape[3]
    out = np.where(den < 1e-30, num / np.sqrt(max(cnt, 1)), num / np.maximum(den, 1e-300))
    return float(out.max()) if out.size else 0.0
