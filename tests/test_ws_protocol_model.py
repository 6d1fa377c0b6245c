"""Model check of the hand-off protocol of the warp-specialised chunk-local
kernel (csrc/kda_chunk_ws.cuh), on the CPU.

An mbarrier wait names the phase it waits for only by its parity, so a waiter
must never fall two phases behind the barrier: it would then take the
current (unfinished) phase for the one it wants and wait for a completion
that only it can cause.  This test runs a model of the kernel's two warp
groups and of the asynchronous completions (TMA copies, MMA commits) under
many random interleavings and checks, at every wait, that the barrier is at
most one phase ahead of the phase waited for, and that every run ends.

The model follows the kernel's order of waits and arrivals per item n
(slot = n mod 2):
  builder: wait raw_full(n); issue raw(n+1); wait a_done[(n-1) mod 2] (item
           n-1); wait b_done[slot] (item n-2); then either issue the [A'; P']
           MMA (commit + arrive on a_done[slot]) or, for a steep item, arrive
           twice;
  solver:  wait a_done[slot] (item n); wait v_full(n); then either issue the
           W^T / U^T MMA (commit on b_done[slot]) and wait for it, or, for a
           steep item, arrive on b_done[slot]; issue V(n+1).
The same model with a single b_done barrier (the form the per-slot barriers
replaced) must fail: that is what the check is for.
"""
import random

NEED = {"raw": 1, "v": 1, "a0": 2, "a1": 2, "b0": 1, "b1": 1}


class Aliased(AssertionError):
    pass


def _run(n_items, steep, seed, per_slot_b=True):
    rnd = random.Random(seed)
    done = {k: 0 for k in NEED}    # completed phases
    arrived = {k: 0 for k in NEED}  # arrivals in the current phase
    pending = ["raw", "v"]          # asynchronous completions in flight (item 0's copies)

    def arrive(bar):
        arrived[bar] += 1
        if arrived[bar] == NEED[bar]:
            arrived[bar] = 0
            done[bar] += 1

    def ready(bar, phase):
        if done[bar] >= phase + 2:
            raise Aliased(f"{bar}: waiting for phase {phase} with {done[bar]} completed")
        return done[bar] == phase + 1

    def b_bar(n):
        return f"b{n & 1}" if per_slot_b else "b0"

    def b_phase(n):
        return n >> 1 if per_slot_b else n

    def builder():
        for n in range(n_items):
            while not ready("raw", n):
                yield
            if n + 1 < n_items:
                pending.append("raw")
            yield
            if n >= 1:
                while not ready(f"a{(n - 1) & 1}", (n - 1) >> 1):
                    yield
            if n >= 2:
                while not ready(b_bar(n - 2), b_phase(n - 2)):
                    yield
            yield
            if steep[n]:
                arrive(f"a{n & 1}")
                arrive(f"a{n & 1}")
            else:
                pending.append(f"a{n & 1}")
                arrive(f"a{n & 1}")
            yield

    def solver():
        for n in range(n_items):
            while not ready(f"a{n & 1}", n >> 1):
                yield
            yield
            while not ready("v", n):
                yield
            if steep[n]:
                arrive(b_bar(n))
            else:
                pending.append(b_bar(n))
                while not ready(b_bar(n), b_phase(n)):
                    yield
            if n + 1 < n_items:
                pending.append("v")
            yield

    groups = {"builder": builder(), "solver": solver()}
    steps = 0
    while groups:
        steps += 1
        if steps > 200000:
            raise AssertionError("no progress: deadlock")
        r = rnd.random()
        if pending and r < 0.3:
            bar = rnd.choice(pending)  # completions of one barrier stay in order
            pending.remove(bar)
            arrive(bar)
            continue
        name = rnd.choice(sorted(groups))
        try:
            next(groups[name])
        except StopIteration:
            del groups[name]
    assert not pending  # every copy and MMA issued was waited for


def _cases(count):
    rnd = random.Random(1234)
    for seed in range(count):
        n = rnd.randint(1, 12)
        frac = rnd.choice([0.0, 0.2, 0.5, 1.0])
        yield n, [rnd.random() < frac for _ in range(n)], seed


def test_per_slot_barriers_never_alias():
    for n, steep, seed in _cases(2000):
        _run(n, steep, seed)


def test_single_b_barrier_aliases():
    failures = 0
    for n, steep, seed in _cases(600):
        try:
            _run(n, steep, seed, per_slot_b=False)
        except Aliased:
            failures += 1
    assert failures > 0
