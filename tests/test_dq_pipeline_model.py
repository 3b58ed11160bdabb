"""A host-side model of fa_dq_kernel's pipeline (csrc/fa_dq.cuh), run under many
random interleavings.

The model has the kernel's three roles, its mbarriers and buffers:
  * the TMA producer loads Q_i/dO_i, then K_0 V_0 K_1 V_1 ... into a ring of
    single-tile slots, waiting on each slot's "empty" barrier;
  * the MMA issuer issues S(0) dP(0) | S(j+1) [wait dS(j)] dQ(j) dP(j+1) | ...
    and commits barriers behind them (a commit arrives once every MMA issued
    before it has completed);
  * the two compute halves read S(j), wait for dP(j), write dS(j) over S(j).
Loads land and MMAs run asynchronously: an MMA starts and completes in issue
order, possibly long after it was issued, and reads its operands from start to
completion.  A wait on an mbarrier is a parity wait, as on the device, and the
model fails if a parity wait could confuse two phases of one barrier.

Checked for every interleaving: no deadlock, no phase aliasing, every MMA
reads the tile it was meant to (the right K_j / V_j in its slot, dS(j) in the
S buffer), no role reads a buffer an MMA is still writing, dQ accumulates the
key tiles in ascending order, and the epilogue sees all of them.
"""
from __future__ import annotations

import random

import pytest


class Bar:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.done = name, count, 0, 0

    def arrive(self):
        self.pending += 1
        assert self.pending <= self.count, self.name
        if self.pending == self.count:
            self.pending, self.done = 0, self.done + 1

    def ready(self, k):
        """Parity wait for phase k (the (k+1)-th completion)."""
        assert self.done <= k + 1, f"{self.name}: waiting for phase {k} after {self.done} completions"
        if self.done < k:
            assert (self.done & 1) == (k & 1), f"{self.name}: a parity wait for phase {k} would pass early"
        return self.done >= k + 1


def simulate(n_kv: int, slots: int, seed: int) -> None:
    rnd = random.Random(seed)
    qdo = Bar("qdo", 1)
    kv_full = [Bar(f"kv_full{s}", 1) for s in range(slots)]
    kv_empty = [Bar(f"kv_empty{s}", 1) for s in range(slots)]
    s_full = [Bar("s_full0", 1), Bar("s_full1", 1)]
    dp_full, ds_full, dq_done, epi = Bar("dp_full", 1), Bar("ds_full", 2), Bar("dq_done", 1), Bar("epi", 2)

    slot = [None] * slots              # tile held by each ring slot
    sbuf = [[None, None], [None, None]]  # S/dS buffer b, column half h
    dp = [None]
    acc = [0]                          # key tiles accumulated into dQ
    busy = set()                       # buffers an MMA is writing
    loads, mmas, commits = [], [], []  # in flight
    issued, completed = [0], [0]

    def issue(kind, j, **kw):
        mmas.append(dict(kind=kind, j=j, started=False, **kw))
        issued[0] += 1

    def commit(bar):
        commits.append((issued[0], bar))

    def producer():
        yield lambda: True
        loads.append(("Q", 0, qdo, None))
        for idx in range(2 * n_kv):
            s, n = idx % slots, idx // slots
            if n > 0:
                yield lambda s=s, n=n: kv_empty[s].ready(n - 1)
            loads.append(("V" if idx & 1 else "K", idx >> 1, kv_full[s], s))

    def issuer():
        def kv(idx):
            return lambda: kv_full[idx % slots].ready(idx // slots)

        def S(j):
            issue("S", j, sk=(2 * j) % slots)
            commit(s_full[j & 1])

        def dP(j):
            sv = (2 * j + 1) % slots
            issue("dP", j, sv=sv)
            commit(dp_full)
            commit(kv_empty[sv])

        def dQ(j):
            sk = (2 * j) % slots
            issue("dQ", j, sk=sk)
            commit(kv_empty[sk])

        yield lambda: qdo.ready(0)
        yield kv(0)
        yield kv(1)
        S(0)
        dP(0)
        for j in range(n_kv):
            if j + 1 < n_kv:
                yield kv(2 * j + 2)
                S(j + 1)
            yield lambda j=j: ds_full.ready(j)
            dQ(j)
            if j + 1 < n_kv:
                yield kv(2 * j + 3)
                dP(j + 1)
        commit(dq_done)

    def compute(h):
        for j in range(n_kv):
            b = j & 1
            yield lambda j=j, b=b: s_full[b].ready(j >> 1)
            assert sbuf[b][h] == ("S", j) and ("S", b) not in busy, (sbuf[b][h], j)
            yield lambda: True  # exponentials
            yield lambda j=j: dp_full.ready(j)
            assert dp[0] == ("dP", j) and "dP" not in busy, (dp[0], j)
            yield lambda: True  # dS
            assert ("S", b) not in busy
            sbuf[b][h] = ("dS", j)
            ds_full.arrive()
        yield lambda: dq_done.ready(0)
        assert acc[0] == n_kv
        epi.arrive()

    agents = [producer(), issuer(), compute(0), compute(1)]
    waits = [None] * len(agents)
    done = [False] * len(agents)
    for _ in range(100000):
        opts = [("agent", a) for a in range(len(agents))
                if not done[a] and (waits[a] is None or waits[a]())]
        if loads:
            opts.append(("load",))
        pending = [m for m in mmas if not m["started"]]
        running = [m for m in mmas if m["started"]]
        if pending:
            opts.append(("start",))
        if running:
            opts.append(("finish",))
        if not opts:
            assert all(done), f"deadlock (roles done: {done})"
            break
        op = rnd.choice(opts)
        if op[0] == "agent":
            a = op[1]
            try:
                waits[a] = next(agents[a])
            except StopIteration:
                done[a] = True
        elif op[0] == "load":
            kind, j, bar, s = loads.pop(rnd.randrange(len(loads)))
            if s is not None:
                slot[s] = (kind, j)
            bar.arrive()
        elif op[0] == "start":
            m = pending[0]
            m["started"] = True
            j = m["j"]
            if m["kind"] == "S":
                assert slot[m["sk"]] == ("K", j)
                busy.add(("S", j & 1))
            elif m["kind"] == "dP":
                assert slot[m["sv"]] == ("V", j)
                busy.add("dP")
            else:
                assert slot[m["sk"]] == ("K", j) and sbuf[j & 1] == [("dS", j), ("dS", j)]
                assert acc[0] == j
        else:
            m = running[0]
            j = m["j"]
            if m["kind"] == "S":
                assert slot[m["sk"]] == ("K", j)
                sbuf[j & 1] = [("S", j), ("S", j)]
                busy.discard(("S", j & 1))
            elif m["kind"] == "dP":
                assert slot[m["sv"]] == ("V", j)
                dp[0] = ("dP", j)
                busy.discard("dP")
            else:
                assert slot[m["sk"]] == ("K", j) and sbuf[j & 1] == [("dS", j), ("dS", j)]
                acc[0] += 1
            mmas.remove(m)
            completed[0] += 1
            while commits and commits[0][0] <= completed[0]:
                commits.pop(0)[1].arrive()
    else:
        raise AssertionError("no progress")
    assert epi.done == 1


@pytest.mark.parametrize("slots", [5, 8])  # the kernel's ring at d = 128 and d = 64
@pytest.mark.parametrize("n_kv", [1, 2, 3, 7, 16])
def test_pipeline_under_random_interleavings(n_kv, slots):
    for seed in range(100):
        simulate(n_kv, slots, seed)


def test_model_detects_a_missing_wait():
    """The model is not vacuous: without the issuer's wait for dS(j), dQ(j)
    can read an S buffer that still holds S(j)."""
    failures = 0
    for seed in range(50):
        try:
            _simulate_without_ds_wait(4, 5, seed)
        except AssertionError:
            failures += 1
    assert failures > 0


def _simulate_without_ds_wait(n_kv, slots, seed):
    """simulate() with the issuer's ds_full wait replaced by no wait."""
    orig = Bar.ready

    def ready(self, k):
        if self.name == "ds_full":
            return True
        return orig(self, k)

    Bar.ready = ready
    try:
        simulate(n_kv, slots, seed)
    finally:
        Bar.ready = orig
