"""Host-side model of fa_dq_kernel's pipeline (csrc/fa_dq.cuh) under random
interleavings (engine: tests/pipeline_model.py).

Roles, as in the kernel:
  * producer: Q_i / dO_i once, then K_0 V_0 K_1 V_1 ... into a ring of
    single-tile slots, each load after the slot's "empty" barrier;
  * issuer (one thread): S(0) dP(0) | S(j+1) [wait dS(j)] dQ(j) dP(j+1) | ...;
    V_j's slot is released by a commit behind dP(j), K_j's behind dQ(j);
  * compute, two column halves: read S(j), wait for dP(j), read it, write dS(j)
    over their half of S(j); then the epilogue reads dQ.
Checked: no deadlock or phase aliasing; every MMA reads the intended tiles
(K_j / V_j in their slots, dS(j) in both halves of its S buffer, dQ holding
tiles 0..j-1), no load lands in a slot an MMA still uses, no role reads a
buffer an MMA is writing, and the epilogue sees dQ summed over every key tile
in ascending order.
"""
from __future__ import annotations

import pytest

from pipeline_model import Bar, Machine


def dq_model(n_kv: int, slots: int, seed: int, skip_ds_wait: bool = False) -> None:
    M = Machine(seed)
    qdo = Bar("qdo", 2)  # one phase: the kernel's expect-tx covers both loads
    kv_full = [Bar(f"kv_full{s}", 1) for s in range(slots)]
    kv_empty = [Bar(f"kv_empty{s}", 1) for s in range(slots)]
    s_full = [Bar("s_full0", 1), Bar("s_full1", 1)]
    dp_full, ds_full, dq_done, epi = Bar("dp_full", 1), Bar("ds_full", 2), Bar("dq_done", 1), Bar("epi", 2)
    M.tag["dQ"] = 0  # key tiles accumulated

    def producer():
        yield lambda: True
        M.load("Q", "Q", qdo)
        M.load("dO", "dO", qdo)
        for idx in range(2 * n_kv):
            s, n = idx % slots, idx // slots
            if n > 0:
                yield lambda s=s, n=n: kv_empty[s].ready(n - 1)
            M.load(("slot", s), ("V" if idx & 1 else "K", idx >> 1), kv_full[s])

    def issuer():
        def kv(idx):
            return lambda: kv_full[idx % slots].ready(idx // slots)

        def S(j):
            b = j & 1
            M.mma("mma", {"Q": "Q", ("slot", (2 * j) % slots): ("K", j)},
                  {("S", b, 0): ("S", j), ("S", b, 1): ("S", j)})
            M.commit("mma", s_full[b])

        def dP(j):
            sv = (2 * j + 1) % slots
            M.mma("mma", {"dO": "dO", ("slot", sv): ("V", j)}, {"dP": ("dP", j)})
            M.commit("mma", dp_full)
            M.commit("mma", kv_empty[sv])

        def dQ(j):
            sk, b = (2 * j) % slots, j & 1
            M.mma("mma", {("S", b, 0): ("dS", j), ("S", b, 1): ("dS", j), ("slot", sk): ("K", j), "dQ": j},
                  {"dQ": j + 1})
            M.commit("mma", kv_empty[sk])

        yield lambda: qdo.ready(0)
        yield kv(0)
        yield kv(1)
        S(0)
        dP(0)
        for j in range(n_kv):
            if j + 1 < n_kv:
                yield kv(2 * j + 2)
                S(j + 1)
            if not skip_ds_wait:
                yield lambda j=j: ds_full.ready(j)
            dQ(j)
            if j + 1 < n_kv:
                yield kv(2 * j + 3)
                dP(j + 1)
        M.commit("mma", dq_done)

    def compute(h):
        for j in range(n_kv):
            b = j & 1
            yield lambda j=j, b=b: s_full[b].ready(j >> 1)
            M.read(("S", b, h), ("S", j))
            yield lambda: True  # the exponentials
            yield lambda j=j: dp_full.ready(j)
            M.read("dP", ("dP", j))
            yield lambda: True  # dS
            M.write(("S", b, h), ("dS", j))
            ds_full.arrive()
        yield lambda: dq_done.ready(0)
        M.read("dQ", n_kv)
        M.write("Q", "dQ staged")  # the epilogue stages dQ in the Q buffer
        epi.arrive()

    M.run([producer(), issuer(), compute(0), compute(1)])
    assert epi.done == 1


@pytest.mark.parametrize("slots", [5, 8])  # the kernel's ring at d = 128 and d = 64
@pytest.mark.parametrize("n_kv", [1, 2, 3, 7, 16])
def test_pipeline_under_random_interleavings(n_kv, slots):
    for seed in range(100):
        dq_model(n_kv, slots, seed)


def test_model_detects_a_missing_wait():
    """Not vacuous: without the issuer's wait for dS(j), dQ(j) can start on an
    S buffer that still holds S(j)."""
    failures = 0
    for seed in range(50):
        try:
            dq_model(4, 5, seed, skip_ds_wait=True)
        except AssertionError:
            failures += 1
    assert failures > 0


def test_model_rings_match_the_kernel():
    """The ring depths this model runs are the kernel's (read from its source)."""
    import os
    import re
    src = open(os.path.join(os.path.dirname(__file__), "..", "io_aware_exact_23_b200", "csrc", "fa_dq.cuh")).read()
    m = re.search(r"kSlots = \(D == 128\) \? (\d+) : (\d+);", src)
    assert m and {int(m.group(1)), int(m.group(2))} == {5, 8}
