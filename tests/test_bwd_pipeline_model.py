"""Host-side model of fa_bwd_kernel's pipeline (csrc/fa_bwd.cuh) under random
interleavings (engine: tests/pipeline_model.py).

One persistent CTA works through a list of units (a unit: one head's key tile
j, with its query tiles); its tiles are numbered across units (t), and every
per-tile barrier phase and stage follows t.  Roles, as in the kernel:
  * producer: hands each unit to the other roles through a two-slot ring (the
    kernel fetches the next unit from a counter); per tile t, Q_t, dO_t, LSE_t,
    D_t into stage t % S (S = 3 stages at d = 64, 2 at d = 128); at d = 64 Q and
    LSE land on one barrier, dO and D on another, which S^T and dP^T wait for
    separately.  With drain
    warps (d = 64) it reloads a stage after its "empty" barrier; in the
    compute-drain layout (d = 128, and every no-dQ instantiation) it frees tile
    t - S's stage itself just before reloading it: it waits for the compute warps'
    staged dQ(t-S) and reduce-adds it (no dQ: it waits for the issuer's commit
    after dK(t-S)), and frees the last S tiles the same way at the end.
    K_j and V_j of a unit load after its first tile, once every MMA of the
    previous unit has completed (the issuer's per-unit commit);
  * issuer (one thread), five MMAs per query tile:
      d = 128:  S^T(t) dP^T(t) [P^T] dV(t) [dS] dK(t) dQ(t)   (dQ in dP^T's columns,
                so dP^T(t+1) waits until the drain has read dQ(t))
      d = 64:   S^T(first) dP^T(first) | [P^T] dV(t) S^T(t+1) [dS] dK(t) dQ(t) dP^T(t+1) | ...
      no dQ (the deterministic mode's instantiation, both d):
                S^T(first) dP^T(first) | [P^T] dV(t) S^T(t+1) [dS] dK(t) dP^T(t+1) | ...
                with dK(t) committing what dQ(t) commits otherwise;
    S^T(t+1) is put in behind dV(t), which reads P^T(t) from the same columns.  A
    unit's first dV and dK overwrite the accumulators, so they wait until the
    previous unit's epilogue has read them -- implied by their waits for P and dS
    of the unit's first tile, which the compute warps produce after that epilogue;
  * eight compute warps (query-column half w, key-row quarter q): read their part
    of S^T, write P^T over it, then read their part of dP^T and write their rows
    of the dS tile in shared memory (after the previous tile's dK / dQ, which
    read it, have completed).  With dropout they first stage the generator's
    draws in their own part of the dS tile (after the same wait).  At d = 128
    they then drain dQ: once dK(t) and dQ(t) completed, read their part of dQ
    out of TMEM (then the issuer may reuse the columns) and stage it in tile t's
    Q (w = 0) or dO (w = 1) stage buffer.  After a unit's last tile: read dV and
    dK out of TMEM, release the accumulators, and stage each through the warp's
    own part of the dS tile for the stores to global memory;
  * d = 64 only, four dQ drain warps: read their rows of dQ out of TMEM, stage
    them in tile t's Q / dO stage buffers, and the leader reduce-adds them into
    the accumulator and hands the stage back to the producer.
Checked: no deadlock or phase aliasing; every MMA reads the intended tiles (of
the intended unit); no load lands in a buffer an MMA uses; no role reads a
buffer being written or writes one an MMA uses; the drain stages each tile's dQ
only after the MMAs reading that stage finished; dK, dV accumulate exactly their
unit's query tiles.
"""
from __future__ import annotations

import pytest

from pipeline_model import Bar, Machine

HALVES, QUARTERS = range(2), range(4)


def parts(name):
    return [(name, w, q) for w in HALVES for q in QUARTERS]


def bwd_model(units, d: int, seed: int, dropout: bool = False, skip: str = "", no_dq: bool = False) -> None:
    """units: the query-tile counts of the units one CTA works through (an int: one unit)."""
    units = [units] if isinstance(units, int) else list(units)
    n_units = len(units)
    first = [sum(units[:u]) for u in range(n_units)]  # global index of each unit's first tile
    M = Machine(seed)
    compute_drain = d == 128 or no_dq  # the kernel's BwdRoles::kComputeDrain
    S = 3 if d == 64 else 2  # the kernel's BwdCfg::kQStages: tile t sits in stage t % S
    bar_kv = Bar("kv", 2)
    # d = 64: Q, LSE on q_full and dO, D on do_full; d = 128: all four on q_full.
    split = d == 64
    q_full = [Bar(f"q_full{s}", 2 if split else 4) for s in range(S)]
    do_full = [Bar(f"do_full{s}", 2) for s in range(S)] if split else q_full
    qdo_empty = [Bar(f"qdo_empty{s}", 1) for s in range(S)]
    # compute-drain layout: every compute warp staged its dQ part; without dQ, the
    # issuer's commit after dK(t) (a per-stage barrier: a wait on it cannot fall two
    # phases behind, unlike one on dkq_done)
    staged = [Bar(f"staged{s}", 1 if no_dq else 8) for s in range(S)]
    s_full, dp_full = Bar("s_full", 1), Bar("dp_full", 1)
    p_full, ds_full = Bar("p_full", 8), Bar("ds_full", 8)
    dkq_done, dq_empty = Bar("dkq_done", 1), Bar("dq_empty", 8 if compute_drain else 4)
    stage = Bar("stage", 4)
    kv_free = Bar("kv_free", 1)  # the issuer's commit after a unit's last MMA
    consumers = 1 + 8 + (0 if compute_drain else 4)  # issuer, compute warps, drain warps
    unit_full = [Bar(f"unit_full{s}", 1) for s in range(2)]
    unit_empty = [Bar(f"unit_empty{s}", consumers) for s in range(2)]
    dq_cols = "dPT" if d == 128 else "dQc"  # dQ's TMEM columns
    done_units = []

    def get_unit(u):
        """A consumer takes unit u (None: no more) from the ring."""
        yield lambda: unit_full[u & 1].ready(u >> 1)
        M.read(("ring", u & 1), u if u < n_units else None)
        unit_empty[u & 1].arrive()

    def load_q(t):
        M.load(("Q", t % S), ("Q", t), q_full[t % S])
        M.load(("L", t % S), ("L", t), q_full[t % S])

    def load_do(t):
        M.load(("dO", t % S), ("dO", t), do_full[t % S])
        M.load(("Dv", t % S), ("Dv", t), do_full[t % S])

    def free_stage(t, reload=None):
        """Compute-drain layout: the producer frees tile t's stage (and loads tile
        `reload` into it) once the reduce-add has read the staged dQ."""
        st = t % S
        if no_dq:
            yield lambda: staged[st].ready(t // S)
            if reload is not None:
                load_q(reload)
                load_do(reload)
            return
        if skip != "staged_wait":
            yield lambda: staged[st].ready(t // S)
        if skip == "early_q_reload" and reload is not None:
            load_q(reload)  # wrong: before the reduce-add has read the Q buffer
        M.read(("Q", st), ("dQ staged", t))  # the reduce-add's read (waited for)
        yield lambda: True
        M.read(("dO", st), ("dQ staged", t))
        if reload is not None:
            if skip != "early_q_reload":
                load_q(reload)
            load_do(reload)

    def producer():
        yield lambda: True
        for u in range(n_units + 1):
            if u >= 2 and skip != "ring_wait":
                yield lambda u=u: unit_empty[u & 1].ready((u >> 1) - 1)
            M.write(("ring", u & 1), u if u < n_units else None)
            unit_full[u & 1].arrive()
            if u == n_units:
                break
            for it in range(units[u]):
                t = first[u] + it
                s, n = t % S, t // S
                if compute_drain and t >= S:
                    yield from free_stage(t - S, reload=t)
                else:
                    if not compute_drain and n > 0:
                        yield lambda s=s, n=n: qdo_empty[s].ready(n - 1)
                    load_q(t)
                    load_do(t)
                if it == 0:
                    # K_j, V_j of this unit: after every MMA of the previous one (a
                    # per-unit barrier: a wait on dkq_done(t-1) could pass early
                    # with three stages, the producer running that far ahead)
                    if u > 0 and skip != "kv_wait":
                        yield lambda u=u: kv_free.ready(u - 1)
                    M.load("K", ("K", u), bar_kv)
                    M.load("V", ("V", u), bar_kv)
        T = first[-1] + units[-1]
        if compute_drain:
            if not no_dq or skip == "tail_waits":  # no dQ: the epilogue itself waits for the last dK
                for t in range(max(T - S, 0), T):
                    yield from free_stage(t)

    def issuer():
        def q_ready(t):
            return lambda: q_full[t % S].ready(t // S)

        def do_ready(t):
            return lambda: do_full[t % S].ready(t // S)

        for u in range(n_units + 1):
            yield from get_unit(u)
            if u == n_units:
                return
            n_it, t0 = units[u], first[u]

            def sT(t):
                M.mma(0, {"K": ("K", u), ("Q", t % S): ("Q", t)}, {p: ("S", t) for p in parts("ST")})
                M.commit(0, s_full)

            def dPT(t):
                M.mma(0, {"V": ("V", u), ("dO", t % S): ("dO", t)}, {p: ("dP", t) for p in parts("dPT")})
                M.commit(0, dp_full)

            def dV(t):
                it = t - t0
                reads = {**{p: ("P", t) for p in parts("ST")}, ("dO", t % S): ("dO", t)}
                if it > 0:
                    reads["dV"] = (u, it)
                M.mma(0, reads, {"dV": (u, it + 1)})

            def dK(t):
                it = t - t0
                reads = {**{p: ("dS", t) for p in parts("dS")}, ("Q", t % S): ("Q", t)}
                if it > 0:
                    reads["dK"] = (u, it)
                M.mma(0, reads, {"dK": (u, it + 1)})
                if no_dq:  # without the dQ product, dK(t) closes the tile and frees its stage
                    M.commit(0, dkq_done)
                    M.commit(0, staged[t % S])

            def dQ(t):
                cols = parts(dq_cols) if d == 128 else [(dq_cols, 0, q) for q in QUARTERS]
                M.mma(0, {**{p: ("dS", t) for p in parts("dS")}, "K": ("K", u)}, {c: ("dQ", t) for c in cols})
                M.commit(0, dkq_done)

            # A unit's first dV and dK overwrite the accumulators the previous unit's
            # epilogue reads; they wait for P and dS of the unit's first tile, which
            # the compute warps produce only after that epilogue: no wait of their own.
            yield lambda: bar_kv.ready(u)
            if no_dq:
                # S^T(first) dP^T(first) | dV(t) S^T(t+1) [dS] dK(t) dP^T(t+1) | ... at both d
                yield q_ready(t0)
                sT(t0)
                yield do_ready(t0)
                dPT(t0)
                for it in range(n_it):
                    t = t0 + it
                    yield lambda t=t: p_full.ready(t)
                    dV(t)
                    if it + 1 < n_it:
                        yield q_ready(t + 1)
                        sT(t + 1)
                    if skip != "ds_wait":
                        yield lambda t=t: ds_full.ready(t)
                    dK(t)
                    if it + 1 < n_it:
                        yield do_ready(t + 1)
                        dPT(t + 1)
            elif d == 128:
                for it in range(n_it):
                    t = t0 + it
                    yield q_ready(t)
                    sT(t)
                    if t > 0:
                        yield lambda t=t: dq_empty.ready(t - 1)
                    if skip != "do_wait":
                        yield do_ready(t)
                    dPT(t)
                    yield lambda t=t: p_full.ready(t)
                    dV(t)
                    if skip != "ds_wait":
                        yield lambda t=t: ds_full.ready(t)
                    dK(t)
                    dQ(t)
            else:
                yield q_ready(t0)
                sT(t0)
                yield do_ready(t0)
                dPT(t0)
                for it in range(n_it):
                    t = t0 + it
                    yield lambda t=t: p_full.ready(t)
                    dV(t)
                    if it + 1 < n_it:
                        yield q_ready(t + 1)
                        sT(t + 1)
                    yield lambda t=t: ds_full.ready(t)
                    dK(t)
                    if t > 0:
                        yield lambda t=t: dq_empty.ready(t - 1)
                    dQ(t)
                    if it + 1 < n_it:
                        yield do_ready(t + 1)
                        dPT(t + 1)
            M.commit(0, kv_free)

    def compute(w, q):
        for u in range(n_units + 1):
            yield from get_unit(u)
            if u == n_units:
                return
            n_it, t0 = units[u], first[u]
            for it in range(n_it):
                t = t0 + it
                s, n = t % S, t // S
                yield lambda t=t, s=s, n=n: s_full.ready(t) and q_full[s].ready(n)
                if dropout:
                    if t > 0 and skip != "draws_wait":
                        yield lambda t=t: dkq_done.ready(t - 1)
                    M.write(("dS", w, q), ("draws", t))  # the warp's own part of the dS tile
                    M.read(("dS", w, q), ("draws", t))
                M.read(("ST", w, q), ("S", t))
                M.read(("L", s), ("L", t))
                M.write(("ST", w, q), ("P", t))
                p_full.arrive()
                yield lambda t=t: dp_full.ready(t)
                if t > 0:  # implied by dp_full(t): dP^T(t) is issued after dQ(t-1)
                    yield lambda t=t: dkq_done.ready(t - 1)
                yield lambda s=s, n=n: do_full[s].ready(n)
                M.read(("dPT", w, q), ("dP", t))
                M.read(("Dv", s), ("Dv", t))
                M.write(("dS", w, q), ("dS", t))
                ds_full.arrive()
                if compute_drain and not no_dq:
                    if skip != "drain_wait":
                        yield lambda t=t: dkq_done.ready(t)
                    M.read((dq_cols, w, q), ("dQ", t))
                    dq_empty.arrive()
                    M.write(("Q" if w == 0 else "dO", s), ("dQ staged", t))
                    staged[s].arrive()
            # epilogue of unit u: dV, dK out of TMEM, then through the warp's part
            # of the dS tile to global memory
            t_last = t0 + n_it - 1
            if skip != "epi_wait":
                yield lambda t=t_last: dkq_done.ready(t)
            M.read("dV", (u, n_it))
            M.read("dK", (u, n_it))
            for what in ("dV out", "dK out"):
                M.write(("dS", w, q), (what, u))
                yield lambda: True
                M.read(("dS", w, q), (what, u))
            done_units.append((u, w, q))

    def drain(q):
        for u in range(n_units + 1):
            yield from get_unit(u)
            if u == n_units:
                return
            for it in range(units[u]):
                t = first[u] + it
                s = t % S
                yield lambda t=t: dkq_done.ready(t)
                M.read((dq_cols, 0, q), ("dQ", t))
                dq_empty.arrive()
                M.write(("Q", s), ("dQ staged", t))
                M.write(("dO", s), ("dQ staged", t))
                stage.arrive()
                if q == 0:  # the leader: reduce-add the staged tile, release the stage
                    yield lambda t=t: stage.ready(t)
                    M.read(("Q", s), ("dQ staged", t))
                    M.read(("dO", s), ("dQ staged", t))
                    qdo_empty[s].arrive()

    roles = [producer(), issuer()] + [compute(w, q) for w in HALVES for q in QUARTERS]
    if not compute_drain:
        roles += [drain(q) for q in QUARTERS]
    M.run(roles)
    assert len(done_units) == 8 * n_units


UNITS = [1, 2, 3, 5, 8, (1, 1, 1), (2, 3), (4, 1, 3), (3, 5, 2, 1)]


@pytest.mark.parametrize("dropout", [False, True])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("units", UNITS, ids=str)
def test_pipeline_under_random_interleavings(units, d, dropout):
    for seed in range(40):
        bwd_model(units, d, seed, dropout=dropout)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("units", UNITS, ids=str)
def test_no_dq_pipeline_under_random_interleavings(units, d):
    """The deterministic mode's instantiation: no dQ product, no dQ drain."""
    for seed in range(40):
        bwd_model(units, d, seed, no_dq=True)


@pytest.mark.parametrize("d,no_dq", [(128, False), (64, False), (128, True)])
def test_unit_handover_needs_its_kv_wait(d, no_dq):
    """Not vacuous across units: loading the next unit's K / V before the previous
    unit's last MMAs completed fails the model.  (Two other handovers need no
    wait of their own, and the model shows it: the ring slot of unit u - 2 is only
    rewritten after every role has taken unit u - 1, since the producer's stage
    reloads depend on their progress; and a unit's first dV / dK follow its first
    P and dS, which the compute warps produce after the previous epilogue read the
    accumulators.  The kernel keeps the ring waits anyway.)"""
    failures = 0
    for seed in range(60):
        try:
            bwd_model((2, 3, 1, 2), d, seed, no_dq=no_dq, skip="kv_wait")
        except AssertionError:
            failures += 1
    assert failures > 0


@pytest.mark.parametrize("d,no_dq", [(64, False), (128, True), (64, True)])
def test_epilogue_needs_the_last_dk_dq(d, no_dq):
    """Not vacuous: an epilogue that reads dK / dV and stages them in the dS tile
    without waiting for the last dK / dQ reads unfinished accumulators.  (At
    d = 128 with dQ the compute warps' own drain already waits for them.)"""
    failures = 0
    for seed in range(40):
        try:
            bwd_model(4, d, seed, no_dq=no_dq, skip="epi_wait")
        except AssertionError:
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


@pytest.mark.parametrize("skip", ["staged_wait", "drain_wait", "early_q_reload"])
def test_compute_drain_model_detects_a_missing_wait(skip):
    """Not vacuous for the compute-drain layout: a producer that reduce-adds and
    reloads a stage without waiting for every warp's staged dQ, or that reloads
    Q before the reduce-add has read it, or compute warps that read dQ before
    dK / dQ completed, fail the model.  (The issuer's wait for dO(t) before
    dP^T(t) has no such control here: dO loads together with Q, which S^T(t)
    waited for, and dP^T(t) also waits for the drain of dQ(t-1).)"""
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
