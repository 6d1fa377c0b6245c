#!/usr/bin/env python
"""Benchmark of the KDA hot path on B200.

Headline: chunkwise prefill tokens/s on B=8, H=32, T=8192, dk=dv=128 (bf16
q/k/v, fp32 gates and state), one prefill call per step, inputs resident in
HBM (2.7 GB of inputs: larger than the 126 MB L2, so no flush is needed).
Beside it, each with its roofline fraction and the fp64 CPU oracle timed on
this host's cores: the other prefill workloads (B1 H2 T256 d32 fp32, B1 H16
T4096 with a random initial state, 16 packed sequences of ~521K tokens), the
recurrent decode (256 sequences x 32 heads, in-place fp32 state, one token per
step) as state GB/s, the Gated DeltaNet variant, the prefill from raw
projections with the input preparation fused in, one long sequence with few
heads (split into segments), the backward pass, and an end-to-end figure
through the C ABI's host-buffer call (pinned host -> device copies, prefill,
copies back, pipelined by the library).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (launched with torch.distributed.run): every rank processes its own
full batch (weak scaling; units are independent, no data-path collective);
timing is the max over ranks of CUDA-event time.

Profiling mode (one operation on a chosen shape, a few calls, for ncu):

    python bench.py --profile-op prefill --B 2 --T 8192 --H 32 --iters 2
    python bench.py --profile-op decode --N 128 --H 32 --iters 2
    python bench.py --profile-op bwd --B 2 --T 1024 --H 32 --iters 2
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import kda_workloads as W  # noqa: E402

METRIC = "KDA prefill tokens/s (B8 H32 T8192 d128) + decode state GB/s, % of roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# Algorithmic work per token-head at dk = dv = 128, C = 64 (minimum traffic:
# q, k, v bf16 + g fp32 + beta fp32 + o bf16; flops of the dense chunk
# contractions A, P, W, U, P.E, W.S, Q.S, K^T.E).
PREFILL_BYTES_PER_TOKEN_HEAD = 3 * 256 + 512 + 4 + 256
PREFILL_FLOPS_PER_TOKEN_HEAD = 6 * 128 * 128 + 2 * 64 * (3 * 128 + 2 * 128)
STATE_BYTES = 128 * 128 * 4
# decode: state read + write, q, k, v, o bf16, g fp32, beta fp32 per head-step
DECODE_BYTES_PER_HEAD_STEP = 2 * STATE_BYTES + 3 * 256 + 512 + 4 + 256
# Gated DeltaNet (one fp32 gate per token-head instead of dk)
GDN_PREFILL_BYTES_PER_TOKEN_HEAD = 3 * 256 + 4 + 4 + 256
GDN_DECODE_BYTES_PER_HEAD_STEP = 2 * STATE_BYTES + 3 * 256 + 4 + 4 + 256


def profiled_traffic(kernel, unit_key):
    """DRAM bytes per unit (token-head or head-step) for `kernel` from its ncu
    summary under profiles/, or None when there is none or when one of the
    kernel's source files changed since the counters were taken (the summary
    lists them, space-separated, with their sha1s)."""
    import glob
    import hashlib
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", f"{kernel}_*.md"))):
        fields = {}
        for line in open(path):
            if ":" in line and not line.startswith(("|", " ", "#")):
                key, _, val = line.partition(":")
                fields[key.strip()] = val.strip()
        src, sha, per = fields.get("source_file"), fields.get("source_sha1"), fields.get(unit_key)
        if not (src and sha and per):
            continue
        srcs, shas = src.split(), sha.split()
        if len(srcs) != len(shas):
            continue
        try:
            cur = [hashlib.sha1(open(os.path.join(ROOT, f), "rb").read()).hexdigest() for f in srcs]
        except OSError:
            continue
        if cur == shas:
            return float(per), os.path.basename(path)
    return None, None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi sampling during the timed region (clocks and throttle reasons)."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, fl in rows for i, f in enumerate(fl) if f.lower() == "active"})
        loaded = [r[0] for r in rows]
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(r[1] for r in rows),
                "samples": len(rows), "reasons": reasons}


def dist_setup(n_gpus):
    if n_gpus <= 1 or "RANK" not in os.environ:
        return 0, 1, 0
    import datetime
    import torch.distributed as dist
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    rank, world = dist.get_rank(), dist.get_world_size()
    local = int(os.environ.get("LOCAL_RANK", rank))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world, device):
    if world <= 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _oracle_cores():
    import oracle
    return oracle.max_threads()


def oracle_rate(w, cores):
    """Token-heads/s of the fp64 oracle on this host's cores for workload w's
    head size (a short calibration run)."""
    import oracle
    cal = W.make_prefill(1, 256, cores, w.dk, w.dv, w.dtype, w.g_mu, w.g_sigma, 0.0, seed=w.seed + 1)
    t0 = time.perf_counter()
    oracle.recurrent(cal["q"], cal["k"], cal["v"], cal["g"], cal["beta"], num_threads=cores)
    return 256 * cores / max(time.perf_counter() - t0, 1e-6)


def oracle_baseline(w, target_s=10.0):
    """Time the fp64 CPU oracle on a bounded sample of prefill workload ``w``
    (same recipe, inputs drawn on the host): whole (sequence, head) units of
    full length, enough for about ``target_s`` seconds on this host's cores,
    or the whole workload when it is smaller.  Packed workloads: the sample's
    units come from sequences picked with a fixed seed."""
    import oracle
    import random
    cores = _oracle_cores()
    rate = oracle_rate(w, cores)
    budget = target_s * rate  # token-heads
    if w.lengths:
        # whole heads of one packed sequence picked with a fixed seed
        pick = random.Random(w.seed).randrange(len(w.lengths))
        L = w.lengths[pick]
        units = int(max(1, min(w.H, budget // L)))
        sample = W.make_prefill(1, L, units, w.dk, w.dv, w.dtype, w.g_mu, w.g_sigma, w.s0_std, seed=w.seed)
        desc = f"{units} heads of packed sequence {pick} ({L} tokens; picked with seed {w.seed})"
        token_heads = units * L
    else:
        total_units = w.B * w.H
        units = int(max(1, min(total_units, budget // w.T)))
        if units >= cores:
            units = units // cores * cores if units < total_units else units
        sample = W.make_prefill(1, w.T, units, w.dk, w.dv, w.dtype, w.g_mu, w.g_sigma, w.s0_std, seed=w.seed)
        whole = units == total_units
        desc = (f"{'all' if whole else units} (sequence, head) units x {w.T} tokens"
                f"{' (the whole workload)' if whole else ''}")
        token_heads = units * w.T
    t0 = time.perf_counter()
    oracle.recurrent(sample["q"], sample["k"], sample["v"], sample["g"], sample["beta"], sample["S0"],
                     num_threads=cores)
    dt = time.perf_counter() - t0
    return {"value": token_heads / dt / w.H, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{desc} of the {w.name} recipe ({token_heads} token-heads, fp64 token-by-token "
                      f"recurrence, {dt:.1f} s); tokens/s = token-heads/s / H"}, dt


def oracle_decode_baseline(w, target_s=6.0):
    """The fp64 oracle on a bounded sample of the decode workload: some of its
    (sequence, head) units, all 1024 steps (run as one prefill per unit, which
    is the same recurrence), reported as state GB/s like the GPU figure."""
    import oracle
    cores = _oracle_cores()
    rate = oracle_rate(w, cores)
    units = int(max(cores, min(w.B * w.H, target_s * rate // w.T)))
    steps = W.make_decode_steps(1, units, w.dk, w.dv, w.T, w.dtype, w.g_mu, w.g_sigma, seed=w.seed)
    S0 = W.make_decode_state(1, units, w.dk, w.dv, w.s0_std, seed=w.seed)
    seq = {n: t.transpose(0, 1) for n, t in steps.items()}  # [1, steps, units, ...]
    t0 = time.perf_counter()
    oracle.recurrent(seq["q"], seq["k"], seq["v"], seq["g"], seq["beta"], S0, num_threads=cores)
    dt = time.perf_counter() - t0
    head_steps = units * w.T
    return {"value": head_steps * 2 * STATE_BYTES / dt / 1e9, "unit": "GB/s (state read+write)",
            "cores": cores, "kind": "oracle", "head_steps_per_s": head_steps / dt,
            "sample": f"{units} of the {w.B * w.H} (sequence, head) units x {w.T} steps of the {w.name} "
                      f"recipe ({head_steps} head-steps, fp64, {dt:.1f} s)"}


def headline_config(w, world):
    """The `config` of the headline line, shared by both arms."""
    return {"workload": w.name, "B": w.B, "T": w.T, "H": w.H, "dk": w.dk, "dv": w.dv,
            "chunk": w.chunk, "g": f"-softplus(N({w.g_mu},{w.g_sigma}))",
            "l2": "inputs (2.7 GB) larger than L2; no flush",
            "parallelism": f"dp{world} (independent batches per GPU)"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = W.PREFILL_B8
    import oracle  # noqa: F401  (built on import of the first call)
    values = []
    total = 0.0
    base = None
    for i in range(args.warmup + args.steps):
        base, dt = oracle_baseline(w, target_s=max(2.0, 60.0 / max(args.steps + args.warmup, 1)))
        if i >= args.warmup:
            values.append(base["value"])
            total += dt
    value = statistics.median(values)
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total / max(args.steps, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": headline_config(w, args.gpus),
            "cpu_baseline": dict(base, value=value),
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def time_launches(fn, steps, stream):
    """CUDA-event time of `steps` calls of fn() on `stream` (ms per call)."""
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(steps):
        fn()
    end.record(stream)
    end.synchronize()
    return start.elapsed_time(end) / steps


def gdn_leg(kda, args, world, dev, stream, peaks):
    """Gated DeltaNet on the headline prefill shape and the decode shape."""
    w = W.GDN_PREFILL_B8
    inp = W.make_workload(w, dev)
    B, T, H, dk, dv = w.B, w.T, w.H, w.dk, w.dv
    o = torch.empty((B, T, H, dv), dtype=torch.bfloat16, device=dev)
    S_out = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    ws = torch.empty(max(kda.workspace_size(B, T, H, dk, dv, 0, w.chunk, torch.bfloat16), 1),
                     dtype=torch.uint8, device=dev)

    def prefill():
        kda.gdn_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["S0"], None, w.chunk,
                          o=o, S_out=S_out, workspace=ws)

    for _ in range(args.warmup):
        prefill()
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(time_launches(prefill, args.steps, stream), world, dev)
    kernel_ms = kda.profile_chunk_fwd(prefill, stream, repeats=max(1, min(args.steps, 5)), dk=dk, dv=dv,
                                      chunk_size=w.chunk, gate="log_token", shape=(B, T, H, 0))
    token_heads = B * T * H
    dom_name, dom_ms = max(kernel_ms.items(), key=lambda kv: kv[1])
    alg_bytes = token_heads * GDN_PREFILL_BYTES_PER_TOKEN_HEAD + B * H * STATE_BYTES
    dom_gbs = alg_bytes / (dom_ms * 1e-3) / 1e9
    prefill_line = {"workload": w.name, "value": world * B * T / (ms * 1e-3), "unit": "tokens/s",
                    "ms_per_step": ms, "kernel_ms": kernel_ms,
                    "roofline": {"bound": "hbm", "kernel": dom_name, "achieved": dom_gbs,
                                 "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": dom_gbs / peaks["hbm_gbs"],
                                 "alg_bytes_per_launch": alg_bytes,
                                 "alg_bytes_rule": "1032 B per token-head (q, k, v, o bf16; one fp32 gate; "
                                                   "beta) + the fp32 final state per unit",
                                 "traffic": None,
                                 "whole_call_frac": alg_bytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"]}}
    del inp, o, S_out, ws
    torch.cuda.empty_cache()

    dw = W.GDN_DECODE
    N, Hd, dd = dw.B, dw.H, dw.dk
    S = W.make_decode_state(N, Hd, dd, dd, dw.s0_std, seed=dw.seed, device=dev)
    xs = W.make_decode_steps(N, Hd, dd, dd, dw.T, dw.dtype, dw.g_mu, dw.g_sigma, seed=dw.seed,
                             device=dev, scalar_gate=True)
    od = torch.empty((N, Hd, dd), dtype=torch.bfloat16, device=dev)
    step = [0]

    def decode_step():
        t = step[0] % dw.T
        kda.gdn_recurrent_step(xs["q"][t], xs["k"][t], xs["v"][t], xs["g"][t], xs["beta"][t], S, o=od)
        step[0] += 1

    for _ in range(16):
        decode_step()
    torch.cuda.synchronize()
    barrier(world)
    dec_ms = max_over_ranks(time_launches(decode_step, dw.T, stream), world, dev)
    heads = N * Hd
    dec_gbs = heads * GDN_DECODE_BYTES_PER_HEAD_STEP / (dec_ms * 1e-3) / 1e9
    decode_line = {"workload": dw.name, "value": world * heads * 2 * STATE_BYTES / (dec_ms * 1e-3) / 1e9,
                   "unit": "GB/s (state read+write)", "us_per_step": dec_ms * 1e3,
                   "roofline": {"bound": "hbm", "achieved": dec_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                "frac": dec_gbs / peaks["hbm_gbs"], "kernel": "kda_decode_step_kernel"}}
    del S, xs, od
    torch.cuda.empty_cache()
    return {"prefill": prefill_line, "decode": decode_line}


def prep_leg(kda, args, world, dev, stream, peaks):
    """KDA from raw projections with the preparation fused into the kernels
    (bf16 gate logits), on the headline shape; beside it the same work done
    unfused (torch elementwise preparation, then kda_chunk_fwd) for contrast."""
    import torch.nn.functional as F
    w = W.PREP_PREFILL_B8
    inp = W.make_workload(w, dev)
    B, T, H, dk, dv = w.B, w.T, w.H, w.dk, w.dv
    o = torch.empty((B, T, H, dv), dtype=torch.bfloat16, device=dev)
    S_out = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    ws = torch.empty(max(kda.workspace_size(B, T, H, dk, dv, 0, w.chunk, torch.bfloat16), 1),
                     dtype=torch.uint8, device=dev)

    def fused():
        kda.chunk_fwd_prep(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"], None, None, w.chunk,
                           o=o, S_out=S_out, workspace=ws)

    def unfused():
        qn = F.normalize(inp["q"].float(), dim=-1).to(torch.bfloat16)
        kn = F.normalize(inp["k"].float(), dim=-1).to(torch.bfloat16)
        g = -F.softplus(inp["a"].float())
        beta = torch.sigmoid(inp["b"])
        kda.chunk_fwd(qn, kn, inp["v"], g, beta, None, None, w.chunk, o=o, S_out=S_out, workspace=ws)

    for fn in (fused, unfused):
        for _ in range(args.warmup):
            fn()
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(time_launches(fused, args.steps, stream), world, dev)
    ms_unfused = max_over_ranks(time_launches(unfused, max(1, min(args.steps, 3)), stream), world, dev)
    kernel_ms = kda.profile_chunk_fwd(fused, stream, repeats=max(1, min(args.steps, 5)), dk=dk, dv=dv,
                                      chunk_size=w.chunk, gate="logit", shape=(B, T, H, 0))
    token_heads = B * T * H
    dom_name, dom_ms = max(kernel_ms.items(), key=lambda kv: kv[1])
    # q, k, v, o bf16 + bf16 gate logits + fp32 beta logit per token-head, + the final state
    alg_bytes = token_heads * (3 * 2 * dk + 2 * dk + 4 + 2 * dv) + B * H * STATE_BYTES
    dom_gbs = alg_bytes / (dom_ms * 1e-3) / 1e9
    line = {"workload": w.name, "value": world * B * T / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms,
            "kernel_ms": kernel_ms,
            "unfused": {"what": "torch normalize/softplus/sigmoid then kda_chunk_fwd", "ms_per_step": ms_unfused,
                        "value": world * B * T / (ms_unfused * 1e-3)},
            "roofline": {"bound": "hbm", "kernel": dom_name, "achieved": dom_gbs, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": dom_gbs / peaks["hbm_gbs"], "alg_bytes_per_launch": alg_bytes,
                         "alg_bytes_rule": "1284 B per token-head (q, k, v, o, gate logits bf16; beta logit "
                                           "fp32) + the fp32 final state per unit",
                         "traffic": None,
                         "whole_call_frac": alg_bytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"]}}
    del inp, o, S_out, ws
    torch.cuda.empty_cache()
    return line


def long_seq_leg(kda, args, world, dev, stream):
    """One long sequence with few heads (B1 H8 T131072): the prefill splits the
    sequence into segments by itself; beside it the same call with segments
    turned off."""
    w = W.LONG_SEQ
    inp = W.make_workload(w, dev)
    B, T, H, dk, dv = w.B, w.T, w.H, w.dk, w.dv
    o = torch.empty((B, T, H, dv), dtype=torch.bfloat16, device=dev)
    S_out = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    out = {"workload": w.name, "unit": "tokens/s"}
    for label, force in (("segmented", 0), ("unsplit", -1)):
        kda.set_segment_chunks(force)
        ws = torch.empty(max(kda.workspace_size(B, T, H, dk, dv, 0, w.chunk, torch.bfloat16), 1),
                         dtype=torch.uint8, device=dev)

        def prefill():
            kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], None, None, w.chunk,
                          o=o, S_out=S_out, workspace=ws)

        for _ in range(args.warmup):
            prefill()
        torch.cuda.synchronize()
        barrier(world)
        ms = max_over_ranks(time_launches(prefill, max(1, min(args.steps, 5)), stream), world, dev)
        out[label] = {"value": world * B * T / (ms * 1e-3), "ms_per_step": ms,
                      "segment_chunks": kda.segment_chunks(B, T, H)}
        del ws
    kda.set_segment_chunks(0)
    del inp, o, S_out
    torch.cuda.empty_cache()
    out["value"] = out["segmented"]["value"]
    return out


def bwd_leg(kda, args, world, dev, stream, peaks):
    """Backward pass on the headline shape: gradients of a loss with a random
    dL/do (bf16) and no final-state term; tokens/s of one kda_chunk_bwd call."""
    w = W.PREFILL_B8
    inp = W.make_workload(w, dev)
    B, T, H, d = w.B, w.T, w.H, w.dk
    gen = torch.Generator(device=dev).manual_seed(w.seed + 77)
    dout = torch.randn(inp["v"].shape, generator=gen, device=dev).to(torch.bfloat16)
    ws = torch.empty(max(int(kda.load_library().kda_chunk_bwd_workspace_size(B, T, H, d, d, 0)), 1),
                     dtype=torch.uint8, device=dev)

    def bwd():
        kda.chunk_bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], dout, None, None, workspace=ws,
                      need_dS0=False)

    bwd()
    torch.cuda.synchronize()
    barrier(world)
    steps = max(1, min(args.steps, 2))
    ms = max_over_ranks(time_launches(bwd, steps, stream), world, dev)
    th = B * T * H
    # must move: q, k, v, do (bf16) + g, beta in; dq, dk, dv, dg (fp32) + dbeta out;
    # plus the fp32 state checkpoint written and read once per 16-token chunk
    alg = th * (4 * 2 * d + 4 * d + 4 + 4 * 4 * d + 4) + 2 * (th // 16) * d * d * 4
    gbs = alg / (ms * 1e-3) / 1e9
    del inp
    torch.cuda.empty_cache()
    line = {"workload": w.name, "value": world * B * T / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms,
            "kernel": "kda_chunk_bwd_kernel<bf16,128>",
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"], "alg_bytes_per_launch": alg, "traffic": None}}

    # the same shape in the Gated DeltaNet form and from raw projections (one
    # timed call each, after one untimed)
    def timed_once(fn):
        fn()
        torch.cuda.synchronize()
        barrier(world)
        return max_over_ranks(time_launches(fn, 1, stream), world, dev)

    gw = W.GDN_PREFILL_B8
    ginp = W.make_workload(gw, dev)
    gms = timed_once(lambda: kda.gdn_chunk_bwd(ginp["q"], ginp["k"], ginp["v"], ginp["g"], ginp["beta"], dout,
                                               None, None, workspace=ws, need_dS0=False))
    line["gdn"] = {"workload": gw.name, "value": world * B * T / (gms * 1e-3), "ms_per_step": gms}
    del ginp, ws
    torch.cuda.empty_cache()
    pw = W.PREP_PREFILL_B8
    pinp = W.make_workload(pw, dev)
    pws = torch.empty(max(int(kda.load_library().kda_chunk_bwd_prep_workspace_size(B, T, H, d, d, 0)), 1),
                      dtype=torch.uint8, device=dev)
    pms = timed_once(lambda: kda.chunk_bwd_prep(pinp["q"], pinp["k"], pinp["v"], pinp["a"], pinp["b"], dout,
                                                None, None, workspace=pws, need_dS0=False))
    line["prep"] = {"workload": pw.name, "value": world * B * T / (pms * 1e-3), "ms_per_step": pms}
    del pinp, pws, dout
    torch.cuda.empty_cache()
    return line


def prefill_roofline(kda, w, ms, kernel_ms, peaks, peak_src, with_state_in):
    """Roofline entry of one prefill workload.  `frac` follows the survey's
    algorithmic bytes: 1,540 B per token-head (q, k, v, o bf16; g fp32; beta)
    plus the fp32 state per (sequence, head) unit (S_out, and S0 when given),
    over the dominant kernel's CUDA-event time.  The whole call's fraction and
    the tensor fraction (dense-contraction flops over the call) sit beside it;
    the dominant kernel's own input/output bytes (which in the two-kernel path
    include the per-chunk image it writes to HBM) are reported separately and
    do not enter `frac`."""
    d = w.dk
    token_heads = w.tokens * w.H
    units = w.num_seqs * w.H
    esz = 2 if w.dtype == "bf16" else 4
    per_th = 3 * d * esz + d * esz + d * 4 + 4  # q, k, v, o; g fp32; beta (1,540 B at d = 128, bf16)
    state = w.dk * w.dv * 4
    alg_bytes = token_heads * per_th + units * state * (2 if with_state_in else 1)
    alg_flops = token_heads * (6 * w.dk * w.dv + 2 * w.chunk * (3 * w.dk + 2 * w.dv))
    dom_name, dom_ms = max(kernel_ms.items(), key=lambda kv: kv[1])
    achieved = alg_bytes / (dom_ms * 1e-3) / 1e9
    per_unit, prof_file = profiled_traffic(dom_name, "traffic_bytes_per_token_head")
    own = kda.algorithmic_bytes_per_launch(dom_name, token_heads, units, d=d, with_state_in=with_state_in)
    return {"bound": "hbm", "kernel": dom_name, "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"],
            "traffic": None if per_unit is None else per_unit * token_heads,
            "traffic_source": None if per_unit is None else
            f"profiles/{prof_file}: DRAM bytes per token-head of a smaller launch x {token_heads} token-heads",
            "alg_bytes_per_launch": alg_bytes,
            "alg_bytes_rule": f"{per_th} B per token-head (q, k, v, o, g, beta) + {state} B fp32 state per "
                              f"unit (S_out, and S0 when given)",
            "peak_source": f"{peak_src} HBM copy bandwidth",
            "whole_call_frac": alg_bytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
            "tensor_frac": alg_flops / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
            "tensor_peak_source": f"{peak_src} cuBLAS bf16 burst",
            "kernel_ms": kernel_ms,
            "dominant_kernel_own_bytes": {"bytes": own, "gbs": own / (dom_ms * 1e-3) / 1e9,
                                          "frac": own / (dom_ms * 1e-3) / 1e9 / peaks["hbm_gbs"]}}


def prefill_leg(kda, w, args, world, dev, stream, peaks, peak_src, sample_clocks=False, cpu=True,
                cpu_target_s=10.0):
    """One prefill workload: tokens/s of kda_chunk_fwd calls on resident
    inputs, the per-phase CUDA-event times, the roofline entry, and (rank 0,
    N = 1) the oracle on a bounded sample of the same recipe."""
    inp = W.make_workload(w, dev)
    B, T, H, dk, dv = w.B, w.T, w.H, w.dk, w.dv
    tdt = w.torch_dtype
    cu = inp.get("cu_seqlens")
    o = torch.empty((B, T, H, dv), dtype=tdt, device=dev)
    S_out = torch.empty((w.num_seqs, H, dk, dv), dtype=torch.float32, device=dev)
    num_seqs = w.num_seqs if cu is not None else 0
    ws_bytes = kda.workspace_size(B, T, H, dk, dv, num_seqs, w.chunk, tdt)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    kernels = kda.chunk_fwd_kernel_sequence(B, T, H, dk, dv, w.chunk, tdt, num_seqs=num_seqs)

    def call():
        kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["S0"], cu, w.chunk,
                      o=o, S_out=S_out, workspace=ws)

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    clk = ClockSampler(dev.index or 0) if sample_clocks else None
    if clk:
        clk.__enter__()
    try:
        ms = time_launches(call, args.steps, stream)
        kernel_ms = kda.profile_chunk_fwd(call, stream, repeats=max(1, min(args.steps, 5)), dk=dk, dv=dv,
                                          chunk_size=w.chunk, dtype=tdt, packed=cu is not None,
                                          shape=(B, T, H, num_seqs))
    finally:
        if clk:
            clk.__exit__(None, None, None)
    torch.cuda.synchronize()
    barrier(world)
    ms_max = max_over_ranks(ms, world, dev)
    line = {"workload": w.name, "value": world * w.tokens / (ms_max * 1e-3), "unit": "tokens/s",
            "ms_per_step": ms_max, "steps": args.steps, "workspace_bytes": ws_bytes,
            "kernels_per_call": kernels,
            "roofline": prefill_roofline(kda, w, ms, kernel_ms, peaks, peak_src, inp["S0"] is not None)}
    if clk:
        line["clocks"] = clk.summary()
    if tdt == torch.bfloat16 and dk == 128:
        # the same calls on the other tensor-core path, for comparison
        other = kda.PATH_TWO_KERNEL if kda.uses_fused_kernel(B, T, H, num_seqs) else kda.PATH_FUSED
        kda.set_prefill_path(other)
        try:
            ws2 = torch.empty(max(kda.workspace_size(B, T, H, dk, dv, num_seqs, w.chunk, tdt), 1),
                              dtype=torch.uint8, device=dev)

            def call2():
                kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["S0"], cu, w.chunk,
                              o=o, S_out=S_out, workspace=ws2)

            for _ in range(args.warmup):
                call2()
            torch.cuda.synchronize()
            barrier(world)
            ms2 = max_over_ranks(time_launches(call2, max(1, min(args.steps, 5)), stream), world, dev)
            line["other_path"] = {"path": "two kernels" if other == kda.PATH_TWO_KERNEL else "single pass",
                                  "ms_per_step": ms2, "value": world * w.tokens / (ms2 * 1e-3)}
            del ws2
        finally:
            kda.set_prefill_path(kda.PATH_AUTO)
    del inp, o, S_out, ws
    torch.cuda.empty_cache()
    if cpu and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"], _ = oracle_baseline(w, cpu_target_s)
    return line


def decode_leg(kda, args, world, dev, stream, peaks, peak_src):
    """1024 in-place decode steps of the decode workload, as state GB/s."""
    dw = W.DECODE
    N, Hd, dd = dw.B, dw.H, dw.dk
    S = W.make_decode_state(N, Hd, dd, dd, dw.s0_std, seed=dw.seed, device=dev)
    nsteps = dw.T
    xs = W.make_decode_steps(N, Hd, dd, dd, nsteps, dw.dtype, dw.g_mu, dw.g_sigma, seed=dw.seed, device=dev)
    od = torch.empty((N, Hd, dd), dtype=torch.bfloat16, device=dev)
    step = [0]

    def decode_step():
        t = step[0] % nsteps
        kda.recurrent_step(xs["q"][t], xs["k"][t], xs["v"][t], xs["g"][t], xs["beta"][t], S, o=od)
        step[0] += 1

    for _ in range(16):
        decode_step()
    torch.cuda.synchronize()
    barrier(world)
    dec_ms = max_over_ranks(time_launches(decode_step, nsteps, stream), world, dev)
    heads = N * Hd
    state_gbs = world * heads * 2 * STATE_BYTES / (dec_ms * 1e-3) / 1e9
    dec_alg_gbs = heads * DECODE_BYTES_PER_HEAD_STEP / (dec_ms * 1e-3) / 1e9
    dec_unit, dec_prof = profiled_traffic("kda_decode_step_kernel", "traffic_bytes_per_head_step")
    line = {"workload": dw.name, "value": state_gbs, "unit": "GB/s (state read+write)",
            "us_per_step": dec_ms * 1e3, "steps": nsteps,
            "roofline": {"bound": "hbm", "achieved": dec_alg_gbs, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": dec_alg_gbs / peaks["hbm_gbs"],
                         "traffic": None if dec_unit is None else dec_unit * heads,
                         "traffic_source": None if dec_unit is None else
                         f"profiles/{dec_prof}: DRAM bytes per head-step x {heads} head-steps",
                         "alg_bytes_per_launch": heads * DECODE_BYTES_PER_HEAD_STEP,
                         "peak_source": f"{peak_src} HBM copy bandwidth",
                         "kernel": "kda_decode_step_kernel"}}
    del S, xs, od
    torch.cuda.empty_cache()
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = oracle_decode_baseline(dw)
    return line


def packed_shard_leg(kda, w, args, world, rank, dev, stream):
    """The packed workload split across the ranks (N > 1 only): each rank
    takes its longest-first share of the sequences (balanced by token count),
    re-packs them contiguously, and runs kda_chunk_fwd on them alone.  The
    time is the max over ranks, so the value is strong scaling of one fixed
    workload; no collective touches the data."""
    if world <= 1:
        return None
    from kimi_delta_attention_31_b200.sharding import rank_share
    inp = W.make_workload(w, dev)
    sub, mine, cu = rank_share(inp, w.lengths, world, rank)
    tokens = cu[-1]
    run = None
    if tokens > 0:
        S0 = sub["S0"]
        cu_t = torch.tensor(cu, dtype=torch.int32, device=dev)
        o = torch.empty((1, tokens, w.H, w.dv), dtype=w.torch_dtype, device=dev)
        S_out = torch.empty((len(mine), w.H, w.dk, w.dv), dtype=torch.float32, device=dev)
        ws = torch.empty(max(kda.workspace_size(1, tokens, w.H, w.dk, w.dv, len(mine), w.chunk, w.torch_dtype), 1),
                         dtype=torch.uint8, device=dev)

        def run():
            kda.chunk_fwd(sub["q"], sub["k"], sub["v"], sub["g"], sub["beta"], S0, cu_t, w.chunk,
                          o=o, S_out=S_out, workspace=ws)
        for _ in range(args.warmup):
            run()
    del inp
    torch.cuda.synchronize()
    barrier(world)
    ms = time_launches(run, max(1, min(args.steps, 5)), stream) if run else 0.0
    ms_max = max_over_ranks(ms, world, dev)
    torch.cuda.synchronize()
    return {"workload": w.name, "split": "sequences, longest first, by token count",
            "value": w.tokens / (ms_max * 1e-3), "unit": "tokens/s", "ms_per_step": ms_max,
            "scaling": "strong", "rank0_sequences": len(mine) if rank == 0 else None}


def e2e_leg(kda, w, args, world, dev, stream):
    """The headline prefill end to end through the C ABI's host-buffer call
    (kda_chunk_fwd_host, wrapped by HostPrefill): every step copies the pinned
    host inputs to the device, runs the prefill and copies o and S_out back."""
    host = W.make_workload(w, "cpu")
    host = {n: (t.pin_memory() if t is not None else None) for n, t in host.items()}
    runner = kda.HostPrefill(host, dev, w.chunk)
    e2e_steps = max(1, min(args.steps, 3))
    runner(host)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(time_launches(lambda: runner(host), e2e_steps, stream), world, dev)
    out = {"value": world * w.tokens / (e2e_ms * 1e-3), "unit": "tokens/s",
           "h2d_bytes_per_step": runner.h2d_bytes(host), "d2h_bytes_per_step": runner.d2h_bytes(),
           "ms_per_step": e2e_ms, "api": "kda_chunk_fwd_host (C ABI), pinned host buffers",
           "pieces": runner.pieces}
    del runner, host
    torch.cuda.empty_cache()
    return out


def run_ours(args):
    import kimi_delta_attention_31_b200 as kda
    rank, world, local = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    peaks, peak_src = load_peaks()
    w = W.PREFILL_B8

    # ---------------- prefill (headline, config 3) ----------------
    head = prefill_leg(kda, w, args, world, dev, stream, peaks, peak_src, sample_clocks=True,
                       cpu_target_s=10.0)
    value, ms_max = head["value"], head["ms_per_step"]
    clocks = head.pop("clocks")
    cpu = head.pop("cpu_baseline", None)
    # ---------------- the other prefill workloads (configs 1, 2, 4) ----------------
    cfg1 = prefill_leg(kda, W.ORACLE_SMALL, args, world, dev, stream, peaks, peak_src, cpu_target_s=3.0)
    cfg2 = prefill_leg(kda, W.PREFILL_H16, args, world, dev, stream, peaks, peak_src, cpu_target_s=5.0)
    cfg4 = prefill_leg(kda, W.PREFILL_VARLEN, args, world, dev, stream, peaks, peak_src, cpu_target_s=8.0)
    cfg4_split = packed_shard_leg(kda, W.PREFILL_VARLEN, args, world, rank, dev, stream)
    if cfg4_split is not None:
        cfg4["split_over_ranks"] = cfg4_split
    # ---------------- end to end through the host-buffer C call ----------------
    e2e = e2e_leg(kda, w, args, world, dev, stream)
    # ---------------- decode (config 5) ----------------
    decode = decode_leg(kda, args, world, dev, stream, peaks, peak_src)
    # ---------------- Gated DeltaNet, fused preparation, long sequence, backward ----------------
    gdn = gdn_leg(kda, args, world, dev, stream, peaks)
    prep = prep_leg(kda, args, world, dev, stream, peaks)
    long_seq = long_seq_leg(kda, args, world, dev, stream)
    bwd = bwd_leg(kda, args, world, dev, stream, peaks)

    gpu_launches = args.steps * len(head["kernels_per_call"])
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": headline_config(w, world),
            "roofline": head["roofline"], "cpu_baseline": cpu, "e2e": e2e,
            "workspace_bytes": head["workspace_bytes"], "kernels_per_call": head["kernels_per_call"],
            "other_path": head.get("other_path"),
            "cfg1": cfg1, "cfg2": cfg2, "cfg4": cfg4, "decode": decode, "gdn": gdn, "prep": prep,
            "long_seq": long_seq, "bwd": bwd,
            "gpu_launches": gpu_launches, "clocks": clocks}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def run_profile_op(args):
    """A few calls of one operation on a chosen shape (seeded synthetic
    inputs, same recipe as the headline), e.g. for an ncu capture; prints the
    mean CUDA-event time per call."""
    import kimi_delta_attention_31_b200 as kda
    kda.set_local_kernel(args.local_kernel)
    if args.prefill_path is not None:
        kda.set_prefill_path(args.prefill_path)
    dev = torch.device("cuda:0")
    if args.profile_op == "prefill":
        inp = W.make_prefill(args.B, args.T, args.H, args.d, args.d, args.dtype, -5.0, 1.5, 0.0, seed=1, device=dev)
        tdt = inp["q"].dtype
        ws_n = kda.workspace_size(args.B, args.T, args.H, args.d, args.d, 0, args.chunk, tdt)
        ws = torch.empty(max(ws_n, 1), dtype=torch.uint8, device=dev)
        o = torch.empty((args.B, args.T, args.H, args.d), dtype=tdt, device=dev)
        S = torch.empty((args.B, args.H, args.d, args.d), dtype=torch.float32, device=dev)
        call = lambda: kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], None, None,
                                     args.chunk, o=o, S_out=S, workspace=ws)
    elif args.profile_op == "decode":
        S = W.make_decode_state(args.N, args.H, args.d, args.d, 0.02, seed=1, device=dev)
        x = W.make_decode_steps(args.N, args.H, args.d, args.d, 1, args.dtype, seed=2, device=dev)
        x = {n: t[0] for n, t in x.items()}
        o = torch.empty((args.N, args.H, args.d), dtype=x["q"].dtype, device=dev)
        call = lambda: kda.recurrent_step(x["q"], x["k"], x["v"], x["g"], x["beta"], S, o=o)
    else:
        inp = W.make_prefill(args.B, args.T, args.H, args.d, args.d, args.dtype, -5.0, 1.5, 0.0, seed=1, device=dev)
        dout = torch.randn(inp["v"].shape, generator=torch.Generator(device=dev).manual_seed(2),
                           device=dev).to(inp["v"].dtype)
        need = int(kda.load_library().kda_chunk_bwd_workspace_size(args.B, args.T, args.H, args.d, args.d, 0))
        ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
        call = lambda: kda.chunk_bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], dout, None, None,
                                     workspace=ws, need_dS0=False)
    call()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(args.iters):
        call()
    end.record()
    end.synchronize()
    print(f"{args.profile_op}: {start.elapsed_time(end) / max(args.iters, 1):.4f} ms per call", flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    prof = ap.add_argument_group("profiling mode")
    prof.add_argument("--profile-op", choices=["prefill", "decode", "bwd"], default=None)
    prof.add_argument("--B", type=int, default=2)
    prof.add_argument("--T", type=int, default=8192)
    prof.add_argument("--N", type=int, default=64)
    prof.add_argument("--H", type=int, default=32)
    prof.add_argument("--d", type=int, default=128)
    prof.add_argument("--chunk", type=int, default=64)
    prof.add_argument("--dtype", choices=["bf16", "f32"], default="bf16")
    prof.add_argument("--iters", type=int, default=3)
    prof.add_argument("--local-kernel", type=int, choices=[0, 1], default=0,
                      help="chunk-local kernel of the two-kernel prefill: 0 warp-specialised, 1 two-CTA")
    prof.add_argument("--prefill-path", type=int, default=None,
                      help="tensor-core prefill path (see kda_set_prefill_path); default: automatic")
    args = ap.parse_args()
    if args.profile_op:
        return run_profile_op(args)
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
