"""Host model of a factorisation worker group's round protocol (csrc/prepare.cu,
the worker loop of chol_persistent_kernel), run under random interleavings.

A group is four warps that meet at named barriers.  Per round r (slot rd = r & 1):
  top      every warp reads the round's task record from slot rd and the
           readiness flag;
  wait     only when the flag is clear: thread 0 polls, writes the outcome,
           barrier A, every warp reads the outcome;
  copies   thread 0 (warp 0) decodes the next claimed task into slot rd ^ 1;
           barrier C;
  products every warp reads the next record (prefetch, early look); warp 0
           writes the readiness flag for the next round; barrier D;
  release  a thread of warp 1 publishes the round's result.
The model checks that every read sees the value the protocol intends: the
round's own task at the top, the next task after barrier C, the flag of the
round before.  A single-slot variant (the record overwritten in place) must
fail, which shows the interleavings reach the race the two slots prevent.
"""
import random

import pytest

WARPS = 4


class Barrier:
    def __init__(self, n):
        self.n, self.count, self.gen = n, 0, 0

    def arrive(self):
        g = self.gen
        self.count += 1
        if self.count == self.n:
            self.count, self.gen = 0, self.gen + 1
        return g

    def passed(self, g):
        return self.gen > g


def run_group(tasks, seed, slots=2):
    """Simulate one group over `tasks` (the numbers its thread 0 claims, in
    order); returns a list of violations."""
    rng = random.Random(seed)
    ntasks = 10 ** 9
    rec = [None, None]
    ready = [0]
    ok = [0]
    rec[0] = tasks[0]
    seq = list(tasks) + [ntasks]
    bars = {k: Barrier(WARPS) for k in "ACD"}
    bad = []

    def warp(w):
        r = 0
        while True:
            rd = (r & 1) if slots == 2 else 0
            nd = (rd ^ 1) if slots == 2 else 0
            t = rec[rd]
            yield
            if t != seq[r]:
                bad.append(("top", w, r, t, seq[r]))
            if t == ntasks:
                return
            rdy = ready[0]
            yield
            if not rdy:
                if w == 0:
                    ok[0] = 1
                g = bars["A"].arrive()
                while not bars["A"].passed(g):
                    yield
                if ok[0] != 1:
                    bad.append(("ok", w, r))
            yield
            if w == 0:
                rec[nd] = seq[r + 1]        # decode of the claimed task
            yield
            g = bars["C"].arrive()
            while not bars["C"].passed(g):
                yield
            nx = rec[nd]
            if nx != seq[r + 1]:
                bad.append(("next", w, r, nx, seq[r + 1]))
            yield
            if w == 0:
                ready[0] = rng.random() < 0.7 and nx != ntasks
            g = bars["D"].arrive()
            while not bars["D"].passed(g):
                yield
            yield
            r += 1

    live = {w: warp(w) for w in range(WARPS)}
    steps = 0
    while live and steps < 200000:
        w = rng.choice(list(live))
        try:
            next(live[w])
        except StopIteration:
            del live[w]
        steps += 1
    if live:
        bad.append(("stuck", sorted(live)))
    return bad


@pytest.mark.parametrize("seed", range(40))
def test_two_slots_every_read_sees_its_record(seed):
    tasks = sorted(random.Random(seed).sample(range(10000), 25))
    assert run_group(tasks, seed) == []


def test_single_slot_races():
    """The planted mistake: one record slot, overwritten while slower warps
    may still read it at the top of a round whose wait was skipped."""
    found = 0
    for seed in range(40):
        tasks = sorted(random.Random(seed).sample(range(10000), 25))
        found += any(b[0] == "top" for b in run_group(tasks, seed, slots=1))
    assert found > 0
