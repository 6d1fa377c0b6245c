"""Run the KDA backward pass on a chosen shape a few times (seeded synthetic
inputs and output gradient), e.g. to profile it with Nsight Compute:

    python -m kimi_delta_attention_31_b200.run_bwd_workload --B 2 --T 1024 --H 32 --iters 2

Prints the mean CUDA-event time per call.
"""
from __future__ import annotations

import argparse
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import kda_workloads as W  # noqa: E402
import kimi_delta_attention_31_b200 as kda  # noqa: E402


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--B", type=int, default=2)
    ap.add_argument("--T", type=int, default=1024)
    ap.add_argument("--H", type=int, default=32)
    ap.add_argument("--d", type=int, default=128)
    ap.add_argument("--dtype", choices=["bf16", "f32"], default="bf16")
    ap.add_argument("--iters", type=int, default=2)
    a = ap.parse_args(argv)
    dev = torch.device("cuda:0")
    inp = W.make_prefill(a.B, a.T, a.H, a.d, a.d, a.dtype, -5.0, 1.5, 0.0, seed=1, device=dev)
    dout = torch.randn(inp["v"].shape, generator=torch.Generator(device=dev).manual_seed(2), device=dev).to(inp["v"].dtype)
    ws = torch.empty(max(int(kda.load_library().kda_chunk_bwd_workspace_size(a.B, a.T, a.H, a.d, a.d, 0)), 1),
                     dtype=torch.uint8, device=dev)
    call = lambda: kda.chunk_bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], dout, None, None,
                                 workspace=ws, need_dS0=False)
    call()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(a.iters):
        call()
    end.record()
    end.synchronize()
    print(f"bwd: {start.elapsed_time(end) / max(a.iters, 1):.4f} ms per call", flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
