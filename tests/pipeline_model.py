"""A small host-side engine for modelling the kernels' pipelines (test infrastructure).

It runs roles (Python generators) against mbarriers, asynchronous TMA loads and
tensor-pipe MMAs, choosing at random which ready event happens next, and checks
every access to a buffer (a shared-memory slot, a tensor-memory region) against
what is in flight:

* ``Bar``: an mbarrier with an arrival count.  ``ready(k)`` is a parity wait
  for phase k (its (k+1)-th completion); it fails the model when a parity wait
  could confuse two phases (the waiter is two or more phases behind or ahead).
* ``Machine.load(res, tag, bar)``: a TMA load into buffer ``res``; it lands at a
  random later time, sets the buffer's content tag and arrives on ``bar``.  It
  may not be issued while an MMA that reads or writes ``res`` is in flight.
* ``Machine.mma(pipe, reads, writes)``: an MMA issued by the thread ``pipe``.
  Each issuing thread's MMAs run one after another in issue order (different
  issuers are not ordered against each other); an accumulating MMA lists its
  accumulator in both ``reads`` and ``writes``.  At its start every buffer in ``reads``
  must hold the expected tag and no load into it may be in flight; the reads must
  still hold at its finish, when the ``writes`` tags are set.
  ``Machine.commit(pipe, bar)`` arrives on ``bar`` once every MMA that thread
  issued before the commit has finished, as tcgen05.commit does.
* ``Machine.read(res, tag)`` / ``Machine.write(res, tag)``: a role's own access
  (tcgen05.ld/st, st.shared, a TMA store's read).  A read needs the expected
  tag and no MMA or load writing the buffer in flight; a write needs no MMA
  or load using the buffer in flight.
* A role yields a predicate to wait on (``lambda: True`` to just yield), and
  is resumed only when the predicate holds.
* Scheduling: each run picks one role (or none) to be slow -- while it is ready
  it is chosen 50 times less often than any other event -- so that runs also
  explore a waiter that falls far behind the barriers it waits on.

``Machine.run`` fails on a deadlock (no role, load or MMA can make progress
before every role has finished) and on any failed check.
"""
from __future__ import annotations

import random
from collections import Counter


class Bar:
    def __init__(self, name: str, count: int):
        self.name, self.count, self.pending, self.done = name, count, 0, 0

    def arrive(self, n: int = 1):
        for _ in range(n):
            self.pending += 1
            assert self.pending <= self.count, f"{self.name}: too many arrivals"
            if self.pending == self.count:
                self.pending, self.done = 0, self.done + 1

    def ready(self, k: int) -> bool:
        assert self.done <= k + 1, f"{self.name}: waiting for phase {k} after {self.done} completions"
        if self.done < k:
            assert (self.done & 1) == (k & 1), f"{self.name}: a parity wait for phase {k} would pass early"
        return self.done >= k + 1


class Machine:
    def __init__(self, seed: int):
        self.rnd = random.Random(seed)
        self.tag = {}
        self.readers = Counter()   # in-flight MMAs reading a buffer
        self.writers = Counter()   # in-flight MMAs writing a buffer
        self.landing = Counter()   # in-flight loads into a buffer
        self.loads = []
        self.pipes = {}            # issuer -> list of [started, reads, writes]
        self.commits = {}          # issuer -> list of (MMAs issued before, bar)
        self.issued = Counter()
        self.finished = Counter()

    # ------------------------------------------------------------ async work
    def load(self, res, tag, bar: Bar):
        assert self.readers[res] == 0 and self.writers[res] == 0, f"load into {res} while an MMA uses it"
        self.landing[res] += 1
        self.loads.append((res, tag, bar))

    def mma(self, pipe, reads: dict, writes: dict):
        for r in reads:
            self.readers[r] += 1
        for w in writes:
            self.writers[w] += 1
        self.pipes.setdefault(pipe, []).append([False, dict(reads), dict(writes)])
        self.issued[pipe] += 1

    def commit(self, pipe, bar: Bar):
        self.commits.setdefault(pipe, []).append((self.issued[pipe], bar))
        self._flush(pipe)

    def _flush(self, pipe):
        q = self.commits.get(pipe, [])
        while q and q[0][0] <= self.finished[pipe]:
            q.pop(0)[1].arrive()

    # ------------------------------------------------------------ role access
    def read(self, res, tag):
        assert self.writers[res] == 0 and self.landing[res] == 0, f"read of {res} while it is being written"
        assert self.tag.get(res) == tag, f"read of {res}: holds {self.tag.get(res)}, expected {tag}"

    def write(self, res, tag):
        assert self.readers[res] == 0 and self.writers[res] == 0 and self.landing[res] == 0, \
            f"write of {res} while an MMA or load uses it"
        self.tag[res] = tag

    # ------------------------------------------------------------ scheduler
    def run(self, roles, max_events: int = 400000):
        waits = [None] * len(roles)
        done = [False] * len(roles)
        slow = self.rnd.randrange(len(roles) + 1)  # len(roles): no slow role
        for _ in range(max_events):
            opts = [("role", a) for a in range(len(roles)) if not done[a] and (waits[a] is None or waits[a]())]
            if self.loads:
                opts.append(("load",))
            for p, q in self.pipes.items():
                if q:
                    opts.append(("finish" if q[0][0] else "start", p))
            if not opts:
                assert all(done), f"deadlock: roles finished {done}"
                return
            op = self.rnd.choices(opts, weights=[0.02 if o == ("role", slow) else 1.0 for o in opts])[0]
            if op[0] == "role":
                a = op[1]
                try:
                    waits[a] = next(roles[a])
                except StopIteration:
                    done[a] = True
            elif op[0] == "load":
                res, tag, bar = self.loads.pop(self.rnd.randrange(len(self.loads)))
                self.landing[res] -= 1
                self.tag[res] = tag
                bar.arrive()
            elif op[0] == "start":
                m = self.pipes[op[1]][0]
                m[0] = True
                for r, t in m[1].items():
                    assert self.landing[r] == 0, f"MMA reads {r} while a load into it is in flight"
                    assert self.tag.get(r) == t, f"MMA reads {r}: holds {self.tag.get(r)}, expected {t}"
            else:
                p = op[1]
                _, reads, writes = self.pipes[p].pop(0)
                for r, t in reads.items():
                    assert self.tag.get(r) == t, f"{r} changed under an MMA reading it"
                    self.readers[r] -= 1
                for w, t in writes.items():
                    self.tag[w] = t
                    self.writers[w] -= 1
                self.finished[p] += 1
                self._flush(p)
        raise AssertionError("no progress within the event limit")
