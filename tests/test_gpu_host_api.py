"""The public host-buffer API (HostPrefill / chunk_fwd_host): pinned host
inputs in, host outputs back.  The batch is pipelined in row groups across
three streams; the results must equal the device-buffer call bit for bit
(units are independent and each is computed by the same kernels)."""
import pytest
import torch

import kimi_delta_attention_31_b200 as kda
import kda_workloads as W

pytestmark = pytest.mark.gpu


def _pinned(inp):
    return {n: (t.pin_memory() if t is not None else None) for n, t in inp.items()}


@pytest.mark.parametrize("pieces", [None, 1, 3])
def test_host_prefill_equals_device_call(cuda_device, pieces):
    host = _pinned(W.make_prefill(5, 200, 4, 128, 128, "bf16", -3.0, 1.0, 0.05, seed=70))
    dev = {n: (t.to(cuda_device) if t is not None else None) for n, t in host.items()}
    o_ref, S_ref = kda.chunk_fwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], dev["S0"], None, 64)
    runner = kda.HostPrefill(host, cuda_device, 64, pieces=pieces)
    for _ in range(2):  # reuse of the device buffers across calls
        o, S = runner(host)
        torch.cuda.current_stream().synchronize()
        assert torch.equal(o, o_ref.cpu()) and torch.equal(S, S_ref.cpu())
    assert runner.h2d_bytes(host) == sum(t.numel() * t.element_size() for t in host.values() if t is not None)


def test_host_prefill_packed_varlen(cuda_device):
    lens = (17, 64, 130, 1)
    host = _pinned(W.make_prefill(1, sum(lens), 2, 128, 128, "bf16", -3.0, 1.0, 0.05, seed=71, lengths=lens))
    dev = {n: (t.to(cuda_device) if t is not None else None) for n, t in host.items()}
    o_ref, S_ref = kda.chunk_fwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], dev["S0"],
                                 dev["cu_seqlens"], 64)
    o, S = kda.chunk_fwd_host(host, 64, cuda_device)
    assert torch.equal(o, o_ref.cpu()) and torch.equal(S, S_ref.cpu())


def test_c_abi_host_call_on_one_stream_fp32(cuda_device):
    """kda_chunk_fwd_host called straight through ctypes, every stage on one
    stream (the fp32-arithmetic path, d = 64): equals the device-buffer call."""
    import ctypes
    host = _pinned(W.make_prefill(3, 90, 2, 64, 64, "f32", -3.0, 1.0, 0.05, seed=72))
    dev = {n: (t.to(cuda_device) if t is not None else None) for n, t in host.items()}
    o_ref, S_ref = kda.chunk_fwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], dev["S0"], None, 32)
    lib = kda.load_library()
    B, T, H, d = 3, 90, 2, 64
    nbytes = int(lib.kda_chunk_fwd_host_buffer_size(B, T, H, d, d, 0, 32, kda.KDA_F32, 2))
    buf = torch.empty(nbytes, dtype=torch.uint8, device=cuda_device)
    o = torch.empty((B, T, H, d), pin_memory=True)
    S = torch.empty((B, H, d, d), pin_memory=True)
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    st = lib.kda_chunk_fwd_host(p(host["q"]), p(host["k"]), p(host["v"]), p(host["g"]), p(host["beta"]),
                                p(host["S0"]), p(o), p(S), None, 0, B, T, H, d, d, 32, kda.KDA_F32, 2,
                                p(buf), nbytes, s, s, s)
    assert st == 0, kda.last_error()
    torch.cuda.current_stream().synchronize()
    assert torch.equal(o, o_ref.cpu()) and torch.equal(S, S_ref.cpu())
