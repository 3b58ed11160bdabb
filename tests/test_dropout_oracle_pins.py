"""Pins of the dropout oracle (oracle/ref_dropout.c), CPU only.

The generator is pinned by the Philox4x32-10 known-answer vectors; the mask by
its documented counter layout, its keep rate and its independence across
offsets; the attention arithmetic by (a) rate 0 reducing exactly to the
pinned dropout-free oracle, (b) a whole-matrix NumPy restatement with the same
mask, (c) central finite differences of the backward, (d) the causal row 0
closed form and (e) unbiasedness over many masks.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import pytest

import oracle
from oracle.ref_numpy import np_fwd

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rnd(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_philox_known_answers():
    kat = json.load(open(os.path.join(GOLDEN, "philox4x32_10_kat.json")))
    for vec in kat["vectors"]:
        ctr = [int(x, 16) for x in vec["counter"]]
        key = [int(x, 16) for x in vec["key"]]
        assert oracle.philox4x32_10(ctr, key) == [int(x, 16) for x in vec["out"]]


def test_mask_follows_the_counter_layout():
    """keep[bh,i,j] is byte (j&3) of word ((j&15)>>2) of Philox((i, j>>4, bh, offset), seed) compared with T."""
    BH, N, seed, offset, rate = 3, 40, 0x0123456789ABCDEF, 7, 0.3
    keep = oracle.dropout_mask(BH, N, seed, offset, rate)
    T = oracle.dropout_threshold(rate)
    rng = np.random.default_rng(1)
    for _ in range(200):
        bh, i, j = int(rng.integers(BH)), int(rng.integers(N)), int(rng.integers(N))
        w = oracle.philox4x32_10([i, j >> 4, bh, offset], [seed & 0xFFFFFFFF, seed >> 32])
        u = (w[(j & 15) >> 2] >> (8 * (j & 3))) & 0xFF
        assert keep[bh, i, j] == (1 if u >= T else 0)


@pytest.mark.parametrize("rate", [0.1, 0.5, 0.9])
def test_keep_rate(rate):
    keep = oracle.dropout_mask(4, 256, 42, 0, rate)
    p = 1.0 - oracle.dropout_threshold(rate) / 256.0
    n = keep.size
    assert abs(keep.mean() - p) <= 5.0 * math.sqrt(p * (1 - p) / n)


def test_masks_differ_across_offsets_and_seeds():
    a = oracle.dropout_mask(2, 64, 5, 0, 0.5)
    b = oracle.dropout_mask(2, 64, 5, 1, 0.5)
    c = oracle.dropout_mask(2, 64, 6, 0, 0.5)
    for x, y in ((a, b), (a, c)):
        agree = (x == y).mean()
        assert 0.45 < agree < 0.55  # independent fair coins agree half the time


def test_threshold_definition():
    assert oracle.dropout_threshold(0.0) == 0
    assert oracle.dropout_threshold(0.5) == 128
    assert oracle.dropout_threshold(0.1) == 25
    assert oracle.dropout_threshold(0.003) == 0  # below 1/256: nothing is dropped
    assert oracle.dropout_threshold(255.0 / 256.0) == 255
    with pytest.raises(ValueError):
        oracle.dropout_threshold(1.0)


@pytest.mark.parametrize("causal", [False, True])
def test_rate_zero_is_the_dropout_free_oracle(causal):
    B, H, N, d = 1, 2, 33, 16
    q, k, v, do = (rnd((B, H, N, d), s) for s in range(4))
    scale = 1 / math.sqrt(d)
    o0, l0 = oracle.ref_fwd(q, k, v, scale, causal)
    o1, l1 = oracle.ref_fwd_dropout(q, k, v, scale, causal, 0.0, 9, 0)
    assert np.abs(o0 - o1).max() <= 1e-12 and np.abs(l0 - l1).max() <= 1e-12
    g0 = oracle.ref_bwd(q, k, v, do, scale, causal)
    g1 = oracle.ref_bwd_dropout(q, k, v, do, scale, causal, 0.0, 9, 0)
    for a, b in zip(g0, g1):
        assert np.abs(a - b).max() <= 1e-10 * max(1.0, np.abs(a).max())


def numpy_dropout(q, k, v, do, scale, causal, rate, seed, offset):
    """Whole-matrix restatement: O = (P o Z) V and the matrix chain rule, with Z from the mask."""
    B, H, N, d = q.shape
    T = oracle.dropout_threshold(rate)
    z = oracle.dropout_mask(B * H, N, seed, offset, rate).reshape(B, H, N, N) * (256.0 / (256.0 - T))
    o_plain, lse, p = np_fwd(q, k, v, scale, causal)
    pz = p * z
    o = pz @ v
    dpt = do @ np.swapaxes(v, -1, -2)
    dp = z * dpt
    D = (p * dp).sum(-1, keepdims=True)
    ds = p * (dp - D)
    dq = scale * ds @ k
    dk = scale * np.swapaxes(ds, -1, -2) @ q
    dv = np.swapaxes(pz, -1, -2) @ do
    return o, lse, (dq, dk, dv)


@pytest.mark.parametrize("causal", [False, True])
def test_c_matches_numpy_restatement(causal):
    B, H, N, d = 2, 2, 45, 8
    q, k, v, do = (rnd((B, H, N, d), 10 + s) for s in range(4))
    scale, rate, seed, offset = 0.35, 0.25, 1234567, 3
    o, lse = oracle.ref_fwd_dropout(q, k, v, scale, causal, rate, seed, offset)
    grads = oracle.ref_bwd_dropout(q, k, v, do, scale, causal, rate, seed, offset)
    o2, lse2, grads2 = numpy_dropout(q, k, v, do, scale, causal, rate, seed, offset)
    assert np.abs(o - o2).max() <= 1e-12 and np.abs(lse - lse2).max() <= 1e-12
    for a, b in zip(grads, grads2):
        assert np.abs(a - b).max() <= 1e-11


def test_finite_differences():
    """The backward is the gradient of L = sum(O * dO) with the mask held fixed."""
    B, H, N, d = 1, 1, 6, 3
    q, k, v, do = (rnd((B, H, N, d), 20 + s) for s in range(4))
    scale, rate, seed, offset, causal = 0.7, 0.4, 99, 1, False
    dq, dk, dv = oracle.ref_bwd_dropout(q, k, v, do, scale, causal, rate, seed, offset)

    def loss(q_, k_, v_):
        o, _ = oracle.ref_fwd_dropout(q_, k_, v_, scale, causal, rate, seed, offset)
        return float((o * do).sum())

    eps = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for idx in [(0, 0, 0, 0), (0, 0, 2, 1), (0, 0, 5, 2), (0, 0, 3, 0)]:
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
            args_m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
            fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            assert abs(fd - g[idx]) <= 1e-6 * max(1.0, abs(fd)), (name, idx, fd, g[idx])


def test_causal_row0_closed_form():
    """Causal row 0 attends only to key 0: O_0 = Z_00 V_0."""
    B, H, N, d = 1, 3, 17, 4
    q, k, v = (rnd((B, H, N, d), 30 + s) for s in range(3))
    rate, seed, offset = 0.5, 77, 2
    o, _ = oracle.ref_fwd_dropout(q, k, v, 0.5, True, rate, seed, offset)
    keep = oracle.dropout_mask(B * H, N, seed, offset, rate)
    inv = 256.0 / (256.0 - oracle.dropout_threshold(rate))
    for h in range(H):
        assert np.array_equal(o[0, h, 0], keep[h, 0, 0] * inv * v[0, h, 0])


def test_unbiased_over_masks():
    """Averaged over many offsets, O with dropout approaches O without it."""
    B, H, N, d = 1, 1, 8, 4
    q, k, v = (rnd((B, H, N, d), 40 + s) for s in range(3))
    o_plain, _ = oracle.ref_fwd(q, k, v, 0.5, False)
    acc = np.zeros_like(o_plain)
    n = 600
    for off in range(n):
        acc += oracle.ref_fwd_dropout(q, k, v, 0.5, False, 0.3, 5, off)[0]
    err = np.abs(acc / n - o_plain).max()
    assert err <= 0.08 * np.abs(v).max()


def test_single_heads_match_the_whole_batch():
    """head0 selects the mask of a head checked on its own (global index b*H + h)."""
    B, H, N, d = 2, 3, 20, 4
    q, k, v, do = (rnd((B, H, N, d), 50 + s) for s in range(4))
    args = (0.6, False, 0.3, 17, 4)
    o, lse = oracle.ref_fwd_dropout(q, k, v, *args)
    g = oracle.ref_bwd_dropout(q, k, v, do, *args)
    for b in range(B):
        for h in range(H):
            sl = lambda x: x[b:b + 1, h:h + 1]  # noqa: E731
            o1, l1 = oracle.ref_fwd_dropout(sl(q), sl(k), sl(v), *args, head0=b * H + h)
            assert np.array_equal(o1[0, 0], o[b, h]) and np.array_equal(l1[0, 0], lse[b, h])
            g1 = oracle.ref_bwd_dropout(sl(q), sl(k), sl(v), sl(do), *args, head0=b * H + h)
            for x1, x in zip(g1, g):
                assert np.array_equal(x1[0, 0], x[b, h])
