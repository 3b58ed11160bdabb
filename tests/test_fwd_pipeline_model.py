"""Host-side model of fa_fwd_kernel's pipeline (csrc/fa_fwd.cuh) under random
interleavings (engine: tests/pipeline_model.py).

One persistent CTA works through a list of units (a unit: a pair of query
tiles k = 0, 1 of one head); barrier phases follow counts over all its units
(K/V loads, and each tile's KV steps).  Roles, as in the kernel:
  * producer: hands each unit to the other roles through a two-slot ring; per
    unit Q_0 (once the previous unit's last S_0 completed), then K / V tiles into
    the ring in the K-ahead order K_0 K_1 V_0 K_2 V_1 ... K_{n-1} V_{n-2} V_{n-1},
    each load after the slot's "empty" barrier (two arrivals: one per issuer),
    with Q_1 right after K_0 (once the previous unit's last S_1 completed);
  * issuer k (its own thread, so its MMAs are ordered only among themselves):
    per KV step j, S_k(j) = Q_k K_j^T, then, once P_k(j) is in TMEM,
    O_k += P_k(j) V_j.  S_k(j+1) goes in behind PV_k(j) without a wait.  A tile
    that stops before step j (causal) still waits for K_j / V_j and releases them;
    after a unit's last S_k it commits "Q_k free";
  * eight softmax warps (lane quarter rq, column half h): per step and tile, read
    their half of S, compute P against the running max, publish the half-row max,
    read the partner warp's, maybe rescale their part of O (after the previous
    PV, a data-dependent choice made at random here, identical for the two warps
    that share rows), write P over their half of S and arrive; at the end of a
    unit exchange the row sums, read O and write it out through the warp's own
    staging area (a unit's first PV overwrites O, but it follows the unit's first
    P, which the warps write after that).
Checked: no deadlock or phase aliasing; each MMA reads the intended tiles (K_j,
V_j in their slots, Q_k and P_k(j) of the right unit, O_k holding steps 0..j-1);
no load lands in a slot an MMA still uses; no warp reads a buffer an MMA is
writing, or overwrites its half-row max before its partner has read it; the
epilogue sees O_k summed over all of tile k's KV steps of its unit.
"""
from __future__ import annotations

import pytest

from pipeline_model import Bar, Machine


def kv_idx_k(j):
    return 0 if j == 0 else 2 * j - 1


def kv_idx_v(j, n):
    return 2 * j + 2 if j + 1 < n else 2 * j + 1


def load_order(n):
    """(is_k, j) of load number idx, as the producer computes it."""
    out = []
    for idx in range(2 * n):
        is_k = idx == 0 or (idx % 2 == 1 and (idx + 1) // 2 < n)
        j = 0 if idx == 0 else ((idx + 1) // 2 if is_k else (n - 1 if idx == 2 * n - 1 else idx // 2 - 1))
        out.append((is_k, j))
    return out


def fwd_model(units, stages: int, seed: int, pv_without_p_wait: bool = False, skip: str = "") -> None:
    """units: per unit the KV steps of its two query tiles, (n_k0, n_k1); a bare
    pair is one unit."""
    units = [tuple(units)] if isinstance(units[0], int) else [tuple(x) for x in units]
    n_units = len(units)
    M = Machine(seed)
    rnd = M.rnd
    bar_q = [Bar("q0", 1), Bar("q1", 1)]
    q_free = [Bar("q_free0", 1), Bar("q_free1", 1)]  # issuer k: its unit's last S_k completed
    kv_full = [Bar(f"kv_full{s}", 1) for s in range(stages)]
    kv_empty = [Bar(f"kv_empty{s}", 2) for s in range(stages)]
    s_full = [Bar(f"s_full{k}", 1) for k in range(2)]
    p_full = [Bar(f"p_full{k}", 8) for k in range(2)]
    pv_done = [Bar(f"pv_done{k}", 1) for k in range(2)]
    bar_x = [[Bar(f"x{k}{q}", 2) for q in range(4)] for k in range(2)]
    bar_l = [[Bar(f"l{k}{q}", 2) for q in range(4)] for k in range(2)]
    unit_full = [Bar(f"unit_full{s}", 1) for s in range(2)]
    unit_empty = [Bar(f"unit_empty{s}", 10) for s in range(2)]  # two issuers, eight softmax warps
    finished = []
    # running counts at the start of each unit: K/V loads, and S steps of each tile
    g0 = [0] * n_units
    cs = [[0, 0] for _ in range(n_units)]
    for u in range(1, n_units):
        g0[u] = g0[u - 1] + 2 * max(units[u - 1])
        cs[u] = [cs[u - 1][k] + units[u - 1][k] for k in range(2)]
    rescale = {(u, k, j, q): (j > 0 and rnd.random() < 0.3)
               for u in range(n_units) for k in range(2) for j in range(max(units[u])) for q in range(4)}
    xm_read = {}  # (k, h, rq) -> last global step of tile k whose half-row max the partner has read

    for n_k in units:  # the producer's load order must put K_j and V_j where the issuers look for them
        n_kv = max(n_k)
        order = load_order(n_kv)
        for j in range(n_kv):
            assert order[kv_idx_k(j)] == (True, j) and order[kv_idx_v(j, n_kv)] == (False, j)

    def get_unit(u):
        yield lambda: unit_full[u & 1].ready(u >> 1)
        M.read(("ring", u & 1), u if u < n_units else None)
        unit_empty[u & 1].arrive()

    def producer():
        yield lambda: True
        for u in range(n_units + 1):
            if u >= 2:
                yield lambda u=u: unit_empty[u & 1].ready((u >> 1) - 1)
            M.write(("ring", u & 1), u if u < n_units else None)
            unit_full[u & 1].arrive()
            if u == n_units:
                return
            n_kv = max(units[u])
            if u > 0 and skip != "q_free":
                yield lambda u=u: q_free[0].ready(u - 1)
            M.load(("Q", 0), ("Q", u, 0), bar_q[0])
            for idx, (is_k, j) in enumerate(load_order(n_kv)):
                g = g0[u] + idx
                s, n = g % stages, g // stages
                if n > 0:
                    yield lambda s=s, n=n: kv_empty[s].ready(n - 1)
                M.load(("slot", s), ("K" if is_k else "V", u, j), kv_full[s])
                if idx == 0:
                    if u > 0 and skip != "q_free":
                        yield lambda u=u: q_free[1].ready(u - 1)
                    M.load(("Q", 1), ("Q", u, 1), bar_q[1])

    def issuer(k):
        for u in range(n_units + 1):
            yield from get_unit(u)
            if u == n_units:
                return
            n_k, n_kv, c = units[u], max(units[u]), cs[u][k]
            yield lambda u=u: bar_q[k].ready(u)
            for j in range(n_kv):
                iK, iV = g0[u] + kv_idx_k(j), g0[u] + kv_idx_v(j, n_kv)
                sK, sV = iK % stages, iV % stages
                yield lambda iK=iK, sK=sK: kv_full[sK].ready(iK // stages)
                if j >= n_k[k]:
                    kv_empty[sK].arrive()
                    yield lambda iV=iV, sV=sV: kv_full[sV].ready(iV // stages)
                    kv_empty[sV].arrive()
                    continue
                M.mma(k, {("Q", k): ("Q", u, k), ("slot", sK): ("K", u, j)}, {part: ("S", u, j) for part in s_parts(k)})
                M.commit(k, s_full[k])
                M.commit(k, kv_empty[sK])
                if j == n_k[k] - 1:
                    M.commit(k, q_free[k])  # Q_k is not read again in this unit
                yield lambda iV=iV, sV=sV: kv_full[sV].ready(iV // stages)
                if not pv_without_p_wait:
                    yield lambda t=c + j: p_full[k].ready(t)
                reads = {**{part: ("P", u, j) for part in s_parts(k)}, ("slot", sV): ("V", u, j)}
                if j > 0:
                    reads[("O", k)] = (u, j)
                M.mma(k, reads, {("O", k): (u, j + 1)})
                M.commit(k, pv_done[k])
                M.commit(k, kv_empty[sV])

    def softmax(rq, h):
        for u in range(n_units + 1):
            yield from get_unit(u)
            if u == n_units:
                break
            n_k, n_kv = units[u], max(units[u])
            for j in range(n_kv):
                for k in range(2):
                    if j >= n_k[k]:
                        continue
                    t = cs[u][k] + j  # tile k's step over all units
                    yield lambda t=t, k=k: s_full[k].ready(t)
                    M.read(("S", k, h, rq), ("S", u, j))
                    key = (k, h, rq)
                    yield lambda: True  # the optimistic exponentials
                    assert t == 0 or xm_read.get(key) == t - 1, f"half-row max {key} overwritten before it was read"
                    M.write(("xm",) + key, t)
                    bar_x[k][rq].arrive()
                    yield lambda t=t, k=k: bar_x[k][rq].ready(t)
                    pkey = (k, h ^ 1, rq)
                    M.read(("xm",) + pkey, t)
                    xm_read[pkey] = t
                    if rescale[(u, k, j, rq)]:
                        yield lambda t=t, k=k: pv_done[k].ready(t - 1)
                        M.read(("O", k), (u, j))
                        M.write(("O", k), (u, j))
                    M.write(("S", k, h, rq), ("P", u, j))
                    p_full[k].arrive()
            last = [cs[u][k] + n_k[k] - 1 for k in range(2)]
            for k in range(2):  # tile 0's epilogue runs while tile 1's last PV does
                if not (skip == "epi_wait" and k == 1):
                    yield lambda k=k, t=last[k]: pv_done[k].ready(t)
                M.write(("ls", k, h, rq), ("sum", u))
                bar_l[k][rq].arrive()
                yield lambda k=k, u=u: bar_l[k][rq].ready(u)
                M.read(("ls", k, h ^ 1, rq), ("sum", u))
                M.read(("O", k), (u, n_k[k]))
                # the warp's own 2 KB of the epilogue staging, in four rounds
                M.write(("epi", h, rq), ("O", u, k))
                yield lambda: True
                M.read(("epi", h, rq), ("O", u, k))
        finished.append((h, rq))

    roles = [producer(), issuer(0), issuer(1)] + [softmax(q, h) for h in range(2) for q in range(4)]
    M.run(roles)
    assert len(finished) == 8


def s_parts(k):
    """S_k's TMEM in the parts the softmax warps own: column half h x lane quarter rq."""
    return [("S", k, h, q) for h in range(2) for q in range(4)]


def tiles(n_all, u, causal):
    """KV steps of the pair u's two query tiles, as the kernel computes them."""
    if causal:
        return (min(2 * u + 1, n_all), min(2 * u + 2, n_all))
    return (n_all, n_all)


CASES = [(1, 0, False), (1, 0, True), (2, 0, True), (3, 1, True), (4, 1, True), (4, 1, False), (7, 3, True),
         (9, 4, True), (6, 2, False)]


@pytest.mark.parametrize("stages", [4, 8])  # the kernel's ring: bf16 at d = 128; d = 64 and e4m3
@pytest.mark.parametrize("n_all,u,causal", CASES, ids=lambda x: str(x))
def test_pipeline_under_random_interleavings(n_all, u, causal, stages):
    n_k = tiles(n_all, u, causal)
    for seed in range(40):
        fwd_model(n_k, stages, seed)


# A persistent CTA's sequence of units (their KV steps per query tile).
UNIT_LISTS = [[(1, 2), (1, 2)], [(7, 8), (1, 2), (3, 4)], [(3, 3), (3, 3), (3, 3)], [(1, 1), (5, 6), (2, 2), (1, 2)],
              [(2, 2)] * 5]


@pytest.mark.parametrize("stages", [4, 8])
@pytest.mark.parametrize("units", UNIT_LISTS, ids=str)
def test_persistent_units_under_random_interleavings(units, stages):
    for seed in range(40):
        fwd_model(units, stages, seed)


def test_persistent_model_detects_an_early_q_reload():
    """Not vacuous: reloading the next unit's Q_k before the previous unit's last
    S_k completed fails the model."""
    failures = 0
    for seed in range(60):
        try:
            fwd_model([(3, 4), (2, 2), (3, 4)], 4, seed, skip="q_free")
        except AssertionError:
            failures += 1
    assert failures > 0


def test_model_detects_a_missing_epilogue_wait():
    """Not vacuous: reading O_1 in the epilogue without waiting for its own last PV
    (only for tile 0's) fails the model."""
    failures = 0
    for seed in range(60):
        try:
            fwd_model([(3, 4), (2, 2)], 4, seed, skip="epi_wait")
        except AssertionError:
            failures += 1
    assert failures > 0


def test_model_detects_a_missing_wait():
    """Not vacuous: a PV issued without waiting for P reads S, not P."""
    failures = 0
    for seed in range(30):
        try:
            fwd_model((4, 4), 4, seed, pv_without_p_wait=True)
        except AssertionError:
            failures += 1
    assert failures > 0


def test_model_rings_match_the_kernel():
    """The ring depths this model runs are the kernel's (read from its source)."""
    import os
    import re
    src = open(os.path.join(os.path.dirname(__file__), "..", "io_aware_exact_23_b200", "csrc", "fa_fwd.cuh")).read()
    m = re.search(r"kStages = \(FP8 \|\| D == 64\) \? (\d+) : (\d+);", src)
    assert m and {int(m.group(1)), int(m.group(2))} == {4, 8}
