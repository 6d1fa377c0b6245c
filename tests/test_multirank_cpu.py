"""The N > 1 path on CPU: two gloo ranks split packed sequences with the LPT
assignment, each runs the (fp64 oracle) recurrence on its own sequences only,
and the union of their results equals one rank doing everything.  The only
collectives are the test's own result gather and a max-over-ranks reduction
of a timing value (as bench.py does)."""
import os
import tempfile

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from kimi_delta_attention_31_b200.sharding import assign_sequences_lpt, packed_subset, rank_share, shard_range


def test_lpt_assignment_partitions_and_balances():
    lengths = [48253, 60938, 9930, 62204, 17831, 26741, 25781, 30314, 61862, 43504, 5706, 11364, 59824,
               26546, 9694, 20506]
    for world in (1, 2, 3, 4, 8):
        owned = assign_sequences_lpt(lengths, world)
        flat = sorted(i for o in owned for i in o)
        assert flat == list(range(len(lengths)))
        loads = [sum(lengths[i] for i in o) for o in owned]
        # LPT bound: no rank exceeds the average by more than the longest sequence
        assert max(loads) <= sum(lengths) / world + max(lengths)
    assert [list(shard_range(10, 4, r)) for r in range(4)] == [[0, 1, 2], [3, 4, 5], [6, 7], [8, 9]]


def _rank_main(rank, world, init_file, lengths, out_file):
    import oracle
    dist.init_process_group("gloo", init_method=f"file://{init_file}", rank=rank, world_size=world)
    try:
        rng = np.random.default_rng(77)
        T = sum(lengths)
        H, d = 2, 8
        q = rng.standard_normal((1, T, H, d))
        k = rng.standard_normal((1, T, H, d))
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
        v = rng.standard_normal((1, T, H, d))
        g = -rng.random((1, T, H, d))
        beta = rng.random((1, T, H))
        # the benchmark's own gathering of a rank's share (torch tensors)
        share, mine, cu = rank_share({"q": torch.from_numpy(q), "k": torch.from_numpy(k), "v": torch.from_numpy(v),
                                      "g": torch.from_numpy(g), "beta": torch.from_numpy(beta), "S0": None},
                                     lengths, world, rank)
        ranges, cu2 = packed_subset(lengths, mine)
        assert cu == cu2 and share["S0"] is None
        idx = np.concatenate([np.arange(a, b) for a, b in ranges]) if ranges else np.zeros(0, int)
        o, S = oracle.recurrent(share["q"].numpy(), share["k"].numpy(), share["v"].numpy(), share["g"].numpy(),
                                share["beta"].numpy(), cu_seqlens=np.array(cu))
        # max over ranks of a per-rank "time", as the benchmark reports it
        t = torch.tensor([float(rank + 1)], dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        payload = [None] * world
        dist.all_gather_object(payload, {"seqs": mine, "idx": idx, "o": o, "S": S, "tmax": t.item()})
        if rank == 0:
            full_o, full_S = oracle.recurrent(q, k, v, g, beta, cu_seqlens=np.cumsum([0] + list(lengths)))
            ok = all(p["tmax"] == float(world) for p in payload)
            for p in payload:
                ok &= np.allclose(p["o"][0], full_o[0, p["idx"]], atol=1e-13)
                for j, s in enumerate(p["seqs"]):
                    ok &= np.allclose(p["S"][j], full_S[s], atol=1e-13)
            covered = sorted(s for p in payload for s in p["seqs"])
            ok &= covered == list(range(len(lengths)))
            with open(out_file, "w") as f:
                f.write("ok" if ok else "mismatch")
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_sequences_without_exchange():
    lengths = [13, 40, 7, 0, 25, 31]
    with tempfile.TemporaryDirectory() as td:
        init_file = os.path.join(td, "init")
        out_file = os.path.join(td, "out")
        mp.start_processes(_rank_main, args=(2, init_file, lengths, out_file), nprocs=2, join=True,
                           start_method="spawn")
        assert open(out_file).read() == "ok"


def test_rank_share_repacks_tokens_and_initial_states():
    """Each rank's share holds exactly its sequences' tokens, in order, and
    their rows of S0; together the shares cover the batch once."""
    lengths = [13, 40, 7, 0, 25, 31]
    T, H, d = sum(lengths), 2, 4
    gen = torch.Generator().manual_seed(5)
    full = {n: torch.randn((1, T, H, d), generator=gen) for n in ("q", "k", "v", "g")}
    full["beta"] = torch.rand((1, T, H), generator=gen)
    full["S0"] = torch.randn((len(lengths), H, d, d), generator=gen)
    starts = np.cumsum([0] + lengths)
    seen = []
    for rank in range(3):
        share, seqs, cu = rank_share(full, lengths, 3, rank)
        assert cu[-1] == sum(lengths[s] for s in seqs) == share["q"].shape[1]
        for j, s_i in enumerate(seqs):
            a, b = starts[s_i], starts[s_i + 1]
            for n in ("q", "k", "v", "g", "beta"):
                assert torch.equal(share[n][:, cu[j]:cu[j + 1]], full[n][:, a:b])
            assert torch.equal(share["S0"][j], full["S0"][s_i])
        seen += seqs
    assert sorted(seen) == list(range(len(lengths)))
