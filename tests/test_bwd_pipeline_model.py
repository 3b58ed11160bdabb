"""Host-side model of fa_bwd_kernel's pipeline (csrc/fa_bwd.cuh) under random
interleavings (engine: tests/pipeline_model.py).

Roles, as in the kernel (one CTA: key tile j, query tiles it = 0 .. n-1):
  * producer: K_j and V_j once; per query tile Q_i, dO_i, LSE_i, D_i into stage
    it % 2.  With drain warps (d = 64) it reloads a stage after its "empty"
    barrier; in the compute-drain layout (d = 128, and every no-dQ instantiation)
    it frees tile i - 2's stage itself just before reloading it: it waits for the
    compute warps' staged dQ(i-2) and reduce-adds it (no dQ: it waits for
    dK(i-2)), and frees the last two tiles the same way after the last load;
  * issuer (one thread), five MMAs per query tile:
      d = 128:  S^T(i) dP^T(i) [P^T] dV(i) [dS] dK(i) dQ(i)   (dQ in dP^T's columns,
                so dP^T(i+1) waits until the drain has read dQ(i))
      d = 64:   S^T(0) dP^T(0) | [P^T] dV(i) S^T(i+1) [dS] dK(i) dQ(i) dP^T(i+1) | ...
      no dQ (the deterministic mode's instantiation, both d):
                S^T(0) dP^T(0) | [P^T] dV(i) S^T(i+1) [dS] dK(i) dP^T(i+1) | ...
                with dK(i) committing what dQ(i) commits otherwise;
    S^T(i+1) is put in behind dV(i), which reads P^T(i) from the same columns;
  * eight compute warps (query-column half w, key-row quarter q): read their part
    of S^T, write P^T over it, then read their part of dP^T and write their rows
    of the dS tile in shared memory (after the previous tile's dK / dQ, which
    read it, have completed).  With dropout they first stage the generator's
    draws in their own part of the dS tile (after the same wait).  At d = 128
    they then drain dQ: once dK(i) and dQ(i) completed, read their part of dQ
    out of TMEM (then the issuer may reuse the columns) and stage it in tile i's
    Q (w = 0) or dO (w = 1) stage buffer;
  * d = 64 only, four dQ drain warps: read their rows of dQ out of TMEM, stage
    them in tile it's Q / dO stage buffers, and the leader reduce-adds them into
    the accumulator and hands the stage back to the producer;
  * epilogue: after the last dK / dQ (and, at d = 128, the warp's own drain),
    dV and dK are staged in V's and K's buffers and stored.
Checked: no deadlock or phase aliasing; every MMA reads the intended tiles;
no load lands in a buffer an MMA uses; no role reads a buffer being written or
writes one an MMA uses; the drain stages each tile's dQ only after the MMAs
reading that stage finished; dK, dV accumulate every query tile.
"""
from __future__ import annotations

import pytest

from pipeline_model import Bar, Machine

HALVES, QUARTERS = range(2), range(4)


def parts(name):
    return [(name, w, q) for w in HALVES for q in QUARTERS]


def bwd_model(n_it: int, d: int, seed: int, dropout: bool = False, skip: str = "", no_dq: bool = False) -> None:
    M = Machine(seed)
    compute_drain = d == 128 or no_dq  # the kernel's BwdRoles::kComputeDrain
    bar_kv = Bar("kv", 2)
    qdo_full = [Bar(f"qdo_full{s}", 4) for s in range(2)]  # Q, dO, LSE, D
    qdo_empty = [Bar(f"qdo_empty{s}", 1) for s in range(2)]
    staged = [Bar(f"staged{s}", 8) for s in range(2)]  # compute-drain layout
    s_full, dp_full = Bar("s_full", 1), Bar("dp_full", 1)
    p_full, ds_full = Bar("p_full", 8), Bar("ds_full", 8)
    dkq_done, dq_empty = Bar("dkq_done", 1), Bar("dq_empty", 8 if compute_drain else 4)
    epi, stage = Bar("epi", 8), Bar("stage", 4)
    M.tag["dK"] = M.tag["dV"] = 0
    dq_cols = "dPT" if d == 128 else "dQc"  # dQ's TMEM columns

    def free_stage(t):
        """Compute-drain layout: the producer frees tile t's stage."""
        st = t & 1
        if no_dq:
            yield lambda: dkq_done.ready(t)
            return
        if skip != "staged_wait":
            yield lambda: staged[st].ready(t >> 1)
        M.read(("Q", st), ("dQ staged", t))  # the reduce-add's read (waited for)
        M.read(("dO", st), ("dQ staged", t))

    def producer():
        yield lambda: True
        M.load("K", "K", bar_kv)
        M.load("V", "V", bar_kv)
        for it in range(n_it):
            s, n = it & 1, it >> 1
            if compute_drain:
                if it >= 2:
                    yield from free_stage(it - 2)
            elif n > 0:
                yield lambda s=s, n=n: qdo_empty[s].ready(n - 1)
            for nm in ("Q", "dO", "L", "Dv"):
                M.load((nm, s), (nm, it), qdo_full[s])
        if compute_drain:
            if not no_dq or skip == "tail_waits":  # no dQ: the epilogue itself waits for the last dK
                for t in range(max(n_it - 2, 0), n_it):
                    yield from free_stage(t)

    def issuer():
        def stage_ready(it):
            return lambda: qdo_full[it & 1].ready(it >> 1)

        def sT(it):
            s = it & 1
            M.mma(0, {"K": "K", ("Q", s): ("Q", it)}, {p: ("S", it) for p in parts("ST")})
            M.commit(0, s_full)

        def dPT(it):
            s = it & 1
            M.mma(0, {"V": "V", ("dO", s): ("dO", it)}, {p: ("dP", it) for p in parts("dPT")})
            M.commit(0, dp_full)

        def dV(it):
            s = it & 1
            M.mma(0, {**{p: ("P", it) for p in parts("ST")}, ("dO", s): ("dO", it), "dV": it}, {"dV": it + 1})

        def dK(it):
            s = it & 1
            M.mma(0, {**{p: ("dS", it) for p in parts("dS")}, ("Q", s): ("Q", it), "dK": it}, {"dK": it + 1})
            if no_dq:  # without the dQ product, dK(i) closes the tile
                M.commit(0, dkq_done)

        def dQ(it):
            cols = parts(dq_cols) if d == 128 else [(dq_cols, 0, q) for q in QUARTERS]
            M.mma(0, {**{p: ("dS", it) for p in parts("dS")}, "K": "K"}, {c: ("dQ", it) for c in cols})
            M.commit(0, dkq_done)

        yield lambda: bar_kv.ready(0)
        if no_dq:
            # S^T(0) dP^T(0) | dV(i) S^T(i+1) [dS] dK(i) dP^T(i+1) | ... at both d
            yield stage_ready(0)
            sT(0)
            dPT(0)
            for it in range(n_it):
                yield lambda it=it: p_full.ready(it)
                dV(it)
                if it + 1 < n_it:
                    yield stage_ready(it + 1)
                    sT(it + 1)
                if skip != "ds_wait":
                    yield lambda it=it: ds_full.ready(it)
                dK(it)
                if it + 1 < n_it:
                    dPT(it + 1)
        elif d == 128:
            for it in range(n_it):
                yield stage_ready(it)
                sT(it)
                if it > 0:
                    yield lambda it=it: dq_empty.ready(it - 1)
                dPT(it)
                yield lambda it=it: p_full.ready(it)
                dV(it)
                if skip != "ds_wait":
                    yield lambda it=it: ds_full.ready(it)
                dK(it)
                dQ(it)
        else:
            yield stage_ready(0)
            sT(0)
            dPT(0)
            for it in range(n_it):
                yield lambda it=it: p_full.ready(it)
                dV(it)
                if it + 1 < n_it:
                    yield stage_ready(it + 1)
                    sT(it + 1)
                yield lambda it=it: ds_full.ready(it)
                dK(it)
                if it > 0:
                    yield lambda it=it: dq_empty.ready(it - 1)
                dQ(it)
                if it + 1 < n_it:
                    dPT(it + 1)

    def compute(w, q):
        for it in range(n_it):
            s, n = it & 1, it >> 1
            yield lambda it=it, s=s, n=n: s_full.ready(it) and qdo_full[s].ready(n)
            if dropout:
                if it > 0 and skip != "draws_wait":
                    yield lambda it=it: dkq_done.ready(it - 1)
                M.write(("dS", w, q), ("draws", it))  # the warp's own part of the dS tile
                M.read(("dS", w, q), ("draws", it))
            M.read(("ST", w, q), ("S", it))
            M.read(("L", s), ("L", it))
            M.write(("ST", w, q), ("P", it))
            p_full.arrive()
            yield lambda it=it: dp_full.ready(it)
            if it > 0:  # implied by dp_full(it): dP^T(i) is issued after dQ(i-1)
                yield lambda it=it: dkq_done.ready(it - 1)
            M.read(("dPT", w, q), ("dP", it))
            M.read(("Dv", s), ("Dv", it))
            M.write(("dS", w, q), ("dS", it))
            ds_full.arrive()
            if compute_drain and not no_dq:
                s = it & 1
                if skip != "drain_wait":
                    yield lambda it=it: dkq_done.ready(it)
                M.read((dq_cols, w, q), ("dQ", it))
                dq_empty.arrive()
                M.write(("Q" if w == 0 else "dO", s), ("dQ staged", it))
                staged[s].arrive()
        if skip != "epi_wait":
            yield lambda: dkq_done.ready(n_it - 1)
        M.read("dV", n_it)
        M.read("dK", n_it)
        # K_j and V_j are dead once every MMA completed: dV is staged in V's buffer,
        # dK in K's, while the last dQ reduce-adds may still read the stage buffers
        M.write("V", "dV staged")
        M.write("K", "dK staged")
        epi.arrive()
        if w == 0 and q == 0:
            yield lambda: epi.ready(0)
            M.read("V", "dV staged")
            M.read("K", "dK staged")

    def drain(q):
        for it in range(n_it):
            s = it & 1
            yield lambda it=it: dkq_done.ready(it)
            if d == 128:
                for w in HALVES:
                    M.read((dq_cols, w, q), ("dQ", it))
            else:
                M.read((dq_cols, 0, q), ("dQ", it))
            dq_empty.arrive()
            M.write(("Q", s), ("dQ staged", it))
            M.write(("dO", s), ("dQ staged", it))
            stage.arrive()
            if q == 0:  # the leader: reduce-add the staged tile, release the stage
                yield lambda it=it: stage.ready(it)
                M.read(("Q", s), ("dQ staged", it))
                M.read(("dO", s), ("dQ staged", it))
                qdo_empty[s].arrive()

    roles = [producer(), issuer()] + [compute(w, q) for w in HALVES for q in QUARTERS]
    if not compute_drain:
        roles += [drain(q) for q in QUARTERS]
    M.run(roles)
    assert epi.done == 1


@pytest.mark.parametrize("dropout", [False, True])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("n_it", [1, 2, 3, 5, 8])
def test_pipeline_under_random_interleavings(n_it, d, dropout):
    for seed in range(40):
        bwd_model(n_it, d, seed, dropout=dropout)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("n_it", [1, 2, 3, 5, 8])
def test_no_dq_pipeline_under_random_interleavings(n_it, d):
    """The deterministic mode's instantiation: no dQ product, no dQ drain."""
    for seed in range(40):
        bwd_model(n_it, d, seed, no_dq=True)


@pytest.mark.parametrize("d,no_dq", [(64, False), (128, True), (64, True)])
def test_epilogue_needs_the_last_dk_dq(d, no_dq):
    """Not vacuous: an epilogue that stages dK / dV in K's and V's buffers without
    waiting for the last dK / dQ overwrites operands an MMA still reads.  (At
    d = 128 with dQ the compute warps' own drain already waits for them.)"""
    failures = 0
    for seed in range(40):
        try:
            bwd_model(4, d, seed, no_dq=no_dq, skip="epi_wait")
        except AssertionError:
            failures += 1
    assert failures > 0


def test_no_dq_tail_waits_would_alias():
    """Why the producer does not wait for dK(n-2) and dK(n-1) at the end without
    dQ: nothing holds dK(n-1) back until that thread has seen dK(n-2), so a slow
    producer's parity wait can fall two phases behind (the model catches it
    through its slow-role scheduling)."""
    failures = 0
    for seed in range(200):
        try:
            bwd_model(5, 128, seed, no_dq=True, skip="tail_waits")
        except AssertionError as e:
            assert "waiting for phase" in str(e)
            failures += 1
    assert failures > 0


def test_no_dq_model_detects_a_missing_wait():
    failures = 0
    for seed in range(40):
        try:
            bwd_model(4, 128, seed, no_dq=True, skip="ds_wait")
        except AssertionError:
            failures += 1
    assert failures > 0


@pytest.mark.parametrize("skip", ["staged_wait", "drain_wait"])
def test_compute_drain_model_detects_a_missing_wait(skip):
    """Not vacuous for the compute-drain layout: a producer that reduce-adds and
    reloads a stage without waiting for every warp's staged dQ, or compute warps
    that read dQ before dK / dQ completed, fail the model."""
    failures = 0
    for seed in range(40):
        try:
            bwd_model(4, 128, seed, skip=skip)
        except AssertionError:
            failures += 1
    assert failures > 0


@pytest.mark.parametrize("d,dropout,skip", [(128, False, "ds_wait"), (64, True, "draws_wait")])
def test_model_detects_a_missing_wait(d, dropout, skip):
    """Not vacuous: without the issuer's wait for dS(i) (d = 128), or the dropout
    path's wait for dK(i-1) / dQ(i-1) before staging its draws in the dS tile
    (d = 64, where S^T(i) is issued ahead of dK(i-1) and dQ(i-1)), an MMA reads
    the wrong contents of the dS tile."""
    failures = 0
    for seed in range(40):
        try:
            bwd_model(4, d, seed, dropout=dropout, skip=skip)
        except AssertionError:
            failures += 1
    assert failures > 0
