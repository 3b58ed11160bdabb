"""Host-side model of fa_fwd_kernel's pipeline (csrc/fa_fwd.cuh) under random
interleavings (engine: tests/pipeline_model.py).

Roles, as in the kernel (one CTA: a pair of query tiles k = 0, 1):
  * producer: Q_0, then K/V tiles into the ring in the K-ahead order
    K_0 K_1 V_0 K_2 V_1 ... K_{n-1} V_{n-2} V_{n-1} (Q_1 right after K_0), each
    load after the slot's "empty" barrier (two arrivals: one per issuer);
  * issuer k (its own thread, so its MMAs are ordered only among themselves):
    per KV step j, S_k(j) = Q_k K_j^T, then, once P_k(j) is in TMEM,
    O_k += P_k(j) V_j.  S_k(j+1) goes in behind PV_k(j) without a wait.  A tile
    that stops before step j (causal) still waits for K_j / V_j and releases them;
  * eight softmax warps (lane quarter rq, column half h): per step and tile, read
    their half of S, publish the half-row max, read the partner warp's, maybe
    rescale their part of O (after the previous PV, a data-dependent choice made
    at random here, identical for the two warps that share rows), write P over
    their half of S and arrive; at the end exchange the row sums, read O and
    stage it (and its residual) in the warp's own part of the idle ring, from
    where the warp itself stores it to global memory.
Checked: no deadlock or phase aliasing; each MMA reads the intended tiles
(K_j, V_j in their slots, P_k(j) in every warp's part of S_k, O_k holding steps
0..j-1); no load lands in a slot an MMA still uses; no warp reads a buffer an
MMA is writing, or overwrites its half-row max before its partner has read it;
the epilogue sees O_k summed over all of tile k's KV steps, and stages it only
in ring slots no load or MMA still uses.
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


def fwd_model(n_k, stages: int, seed: int, pv_without_p_wait: bool = False) -> None:
    n_kv = max(n_k)
    M = Machine(seed)
    rnd = M.rnd
    bar_q = [Bar("q0", 1), Bar("q1", 1)]
    kv_full = [Bar(f"kv_full{s}", 1) for s in range(stages)]
    kv_empty = [Bar(f"kv_empty{s}", 2) for s in range(stages)]
    s_full = [Bar(f"s_full{k}", 1) for k in range(2)]
    p_full = [Bar(f"p_full{k}", 8) for k in range(2)]
    pv_done = [Bar(f"pv_done{k}", 1) for k in range(2)]
    bar_x = [[Bar(f"x{k}{q}", 2) for q in range(4)] for k in range(2)]
    bar_l = [[Bar(f"l{k}{q}", 2) for q in range(4)] for k in range(2)]
    finished = []
    for k in range(2):
        M.tag[("O", k)] = 0
    rescale = {(k, j, q): (j > 0 and rnd.random() < 0.3) for k in range(2) for j in range(n_kv) for q in range(4)}
    xm_read = {}  # (k, h, rq) -> last step whose half-row max the partner has read

    # the producer's load order must put K_j and V_j where the issuers look for them
    order = load_order(n_kv)
    for j in range(n_kv):
        assert order[kv_idx_k(j)] == (True, j) and order[kv_idx_v(j, n_kv)] == (False, j)

    def producer():
        yield lambda: True
        M.load(("Q", 0), "Q0", bar_q[0])
        for idx, (is_k, j) in enumerate(order):
            s, n = idx % stages, idx // stages
            if n > 0:
                yield lambda s=s, n=n: kv_empty[s].ready(n - 1)
            M.load(("slot", s), ("K" if is_k else "V", j), kv_full[s])
            if idx == 0:
                M.load(("Q", 1), "Q1", bar_q[1])

    def issuer(k):
        yield lambda: bar_q[k].ready(0)
        for j in range(n_kv):
            iK, iV = kv_idx_k(j), kv_idx_v(j, n_kv)
            sK, sV = iK % stages, iV % stages
            yield lambda iK=iK, sK=sK: kv_full[sK].ready(iK // stages)
            if j >= n_k[k]:
                kv_empty[sK].arrive()
                yield lambda iV=iV, sV=sV: kv_full[sV].ready(iV // stages)
                kv_empty[sV].arrive()
                continue
            M.mma(k, {("Q", k): f"Q{k}", ("slot", sK): ("K", j)}, {part: ("S", j) for part in s_parts(k)})
            M.commit(k, s_full[k])
            M.commit(k, kv_empty[sK])
            yield lambda iV=iV, sV=sV: kv_full[sV].ready(iV // stages)
            if not pv_without_p_wait:
                yield lambda j=j: p_full[k].ready(j)
            M.mma(k, {**{part: ("P", j) for part in s_parts(k)}, ("slot", sV): ("V", j), ("O", k): j},
                  {("O", k): j + 1})
            M.commit(k, pv_done[k])
            M.commit(k, kv_empty[sV])

    def softmax(rq, h):
        for j in range(n_kv):
            for k in range(2):
                if j >= n_k[k]:
                    continue
                yield lambda j=j, k=k: s_full[k].ready(j)
                M.read(("S", k, h, rq), ("S", j))
                key = (k, h, rq)
                assert j == 0 or xm_read.get(key) == j - 1, f"half-row max {key} overwritten before it was read"
                M.write(("xm",) + key, j)
                bar_x[k][rq].arrive()
                yield lambda: True  # the optimistic exponentials
                yield lambda j=j, k=k: bar_x[k][rq].ready(j)
                pkey = (k, h ^ 1, rq)
                M.read(("xm",) + pkey, j)
                xm_read[pkey] = j
                if rescale[(k, j, rq)]:
                    yield lambda j=j, k=k: pv_done[k].ready(j - 1)
                    M.read(("O", k), j)
                    M.write(("O", k), j)
                M.write(("S", k, h, rq), ("P", j))
                p_full[k].arrive()
        yield lambda: pv_done[0].ready(n_k[0] - 1) and pv_done[1].ready(n_k[1] - 1)
        for k in range(2):
            M.write(("ls", k, h, rq), "sum")
            bar_l[k][rq].arrive()
            yield lambda k=k: bar_l[k][rq].ready(0)
            M.read(("ls", k, h ^ 1, rq), "sum")
            M.read(("O", k), n_k[k])
            # the warp's 2 x 32 x d bytes of staging: warp 4h + rq, four warps per
            # ring slot at d = 128 (bf16, 4 slots) and d = 64 (8 slots)
            M.write(("slot", h), "epilogue staging")
            M.write(("staging", h, rq), ("O", k))
            yield lambda: True
            M.read(("staging", h, rq), ("O", k))
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
