"""Run the KDA prefill or decode on a chosen shape a few times (seeded
synthetic inputs), e.g. to profile one kernel with Nsight Compute:

    python -m kimi_delta_attention_31_b200.run_workload --op prefill --B 2 --T 8192 --H 32 --iters 3
    python -m kimi_delta_attention_31_b200.run_workload --op prefill --B 2 --T 8192 --H 32 --local-kernel 1
    python -m kimi_delta_attention_31_b200.run_workload --op decode --N 64 --H 32 --iters 5

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
    ap.add_argument("--op", choices=["prefill", "decode"], default="prefill")
    ap.add_argument("--B", type=int, default=2)
    ap.add_argument("--T", type=int, default=8192)
    ap.add_argument("--N", type=int, default=64)
    ap.add_argument("--H", type=int, default=32)
    ap.add_argument("--d", type=int, default=128)
    ap.add_argument("--chunk", type=int, default=64)
    ap.add_argument("--dtype", choices=["bf16", "f32"], default="bf16")
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--local-kernel", type=int, choices=[0, 1], default=0,
                    help="chunk-local kernel of the prefill: 0 warp-specialised (default), 1 two-CTA")
    a = ap.parse_args(argv)
    kda.set_local_kernel(a.local_kernel)
    dev = torch.device("cuda:0")
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if a.op == "prefill":
        inp = W.make_prefill(a.B, a.T, a.H, a.d, a.d, a.dtype, -5.0, 1.5, 0.0, seed=1, device=dev)
        ws_n = kda.workspace_size(a.B, a.T, a.H, a.d, a.d, 0, a.chunk,
                                  torch.bfloat16 if a.dtype == "bf16" else torch.float32)
        ws = torch.empty(max(ws_n, 1), dtype=torch.uint8, device=dev)
        o = torch.empty((a.B, a.T, a.H, a.d), dtype=inp["q"].dtype, device=dev)
        S = torch.empty((a.B, a.H, a.d, a.d), dtype=torch.float32, device=dev)
        call = lambda: kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], None, None,
                                     a.chunk, o=o, S_out=S, workspace=ws)
    else:
        S = W.make_decode_state(a.N, a.H, a.d, a.d, 0.02, seed=1, device=dev)
        x = W.make_decode_steps(a.N, a.H, a.d, a.d, 1, a.dtype, seed=2, device=dev)
        x = {n: t[0] for n, t in x.items()}
        o = torch.empty((a.N, a.H, a.d), dtype=x["q"].dtype, device=dev)
        call = lambda: kda.recurrent_step(x["q"], x["k"], x["v"], x["g"], x["beta"], S, o=o)
    call()
    torch.cuda.synchronize()
    start.record()
    for _ in range(a.iters):
        call()
    end.record()
    end.synchronize()
    print(f"{a.op}: {start.elapsed_time(end) / max(a.iters, 1):.4f} ms per call", flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
