"""Pins for the CPU fp64 oracle: checks that do not come from the oracle itself.

Every pin is a function of a forward callable ``fwd(q, k, v, scale, causal) ->
(O, LSE)`` and a backward callable ``bwd(q, k, v, dO, scale, causal) -> (dQ,
dK, dV)`` on fp64 arrays [B, H, N, d].  The C oracle must pass them all.  To
show the pins have teeth, ``test_planted_mistakes_are_caught`` runs them on
copies of the NumPy restatement with one mistake planted each (a dropped
scale, a transposed operand, a wrong mask, a dropped term, a sign flip ...)
and requires every mutant to fail at least one pin.

Sources of truth, none of them the oracle's own formula retyped:
  * hand-derived 2x2 worked examples (tests/golden/two_by_two.json);
  * closed forms: N = 1 gives O = V; identical keys give O = mean(V) and
    LSE = s + ln N; causal row 0 gives O_0 = V_0; V = 1 gives O = 1; scale = 0
    gives the (prefix) mean of V;
  * invariants: softmax rows sum to 1 (V = identity exposes P); joint K/V row
    permutation leaves O unchanged and a Q permutation permutes O; adding u to
    every key leaves O unchanged and shifts LSE_i by scale*q_i.u;
  * gradient identities: sum_j dK_j = 0, sum_j dV_j = sum_i dO_i and
    sum_i Q_i.dQ_i = sum_j K_j.dK_j;
  * brute force: central finite differences of L = sum(O * dO);
  * a library routine: torch's scaled_dot_product_attention in fp64 on the CPU
    and its autograd gradients.
"""
from __future__ import annotations

import json
import os

import numpy as np
import pytest

import oracle
from oracle import ref_numpy

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def c_fwd(q, k, v, scale, causal):
    return oracle.ref_fwd(q, k, v, scale, causal, nthreads=4)


def c_bwd(q, k, v, dO, scale, causal):
    return oracle.ref_bwd(q, k, v, dO, scale, causal, nthreads=4)


def rnd(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def close(a, b, tol=1e-10):
    a, b = np.asarray(a), np.asarray(b)
    return a.shape == b.shape and np.allclose(a, b, rtol=tol, atol=tol)


# ------------------------------------------------------------------ pins

def pin_golden(fwd, bwd):
    with open(os.path.join(GOLDEN, "two_by_two.json")) as f:
        g = json.load(f)
    for c in g["cases"]:
        t = {nm: np.array(c[nm], dtype=np.float64)[None, None] for nm in ("q", "k", "v", "do")}
        o, lse = fwd(t["q"], t["k"], t["v"], c["scale"], c["causal"])
        dq, dk, dv = bwd(t["q"], t["k"], t["v"], t["do"], c["scale"], c["causal"])
        for nm, got in (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv)):
            want = np.array(c[nm])[None, None]
            if not close(got, want, 1e-12):
                return f"{c['name']}: {nm} {np.asarray(got).ravel()} != {want.ravel()}"
    return None


def pin_n1(fwd, bwd):
    for causal in (False, True):
        q, k, v, dO = (rnd((2, 3, 1, 5), s) for s in range(4))
        o, lse = fwd(q, k, v, 0.7, causal)
        if not close(o, v):
            return "N=1: O != V"
        if not close(lse, 0.7 * (q * k).sum(-1)):
            return "N=1: LSE != scale q.k"
        dq, dk, dv = bwd(q, k, v, dO, 0.7, causal)
        if not (close(dq, 0 * q) and close(dk, 0 * k) and close(dv, dO)):
            return "N=1: gradients"
    return None


def pin_identical_keys(fwd, bwd):
    B, H, N, d = 1, 2, 7, 4
    q = rnd((B, H, N, d), 1)
    k = np.broadcast_to(rnd((B, H, 1, d), 2), (B, H, N, d)).copy()
    v = rnd((B, H, N, d), 3)
    sc = 0.6
    s = sc * np.einsum("bhid,bhd->bhi", q, k[:, :, 0])
    o, lse = fwd(q, k, v, sc, False)
    if not close(o, np.broadcast_to(v.mean(axis=2, keepdims=True), o.shape)):
        return "identical keys: O != mean(V)"
    if not close(lse, s + np.log(N)):
        return "identical keys: LSE != s + ln N"
    o, lse = fwd(q, k, v, sc, True)
    prefix = np.cumsum(v, axis=2) / np.arange(1, N + 1)[None, None, :, None]
    if not close(o, prefix):
        return "identical keys, causal: O != prefix mean"
    if not close(lse, s + np.log(np.arange(1, N + 1))[None, None]):
        return "identical keys, causal: LSE"
    return None


def pin_rows_sum_to_one(fwd, bwd):
    N = 6
    q, k = rnd((1, 2, N, 3), 4), rnd((1, 2, N, 3), 5)
    # d must equal N for V = I; pad Q and K with zero columns (scores unchanged)
    qp = np.concatenate([q, np.zeros((1, 2, N, N - 3))], axis=-1)
    kp = np.concatenate([k, np.zeros((1, 2, N, N - 3))], axis=-1)
    eye = np.broadcast_to(np.eye(N), (1, 2, N, N)).copy()
    for causal in (False, True):
        p, _ = fwd(qp, kp, eye, 0.9, causal)
        if not close(p.sum(-1), np.ones((1, 2, N))):
            return "rows of P do not sum to 1"
        if (p < 0).any():
            return "negative probability"
        if causal and not close(np.triu(p[0, 0], 1), np.zeros((N, N))):
            return "causal P has mass above the diagonal"
        if not causal and (p <= 0).any():
            return "non-causal P has a zero entry"
    return None


def pin_permutations(fwd, bwd):
    B, H, N, d = 2, 2, 9, 4
    q, k, v = rnd((B, H, N, d), 6), rnd((B, H, N, d), 7), rnd((B, H, N, d), 8)
    o, lse = fwd(q, k, v, 0.5, False)
    perm = np.random.default_rng(9).permutation(N)
    o2, lse2 = fwd(q, k[:, :, perm], v[:, :, perm], 0.5, False)
    if not (close(o, o2) and close(lse, lse2)):
        return "joint K/V permutation changed the result"
    o3, lse3 = fwd(q[:, :, perm], k, v, 0.5, False)
    if not (close(o3, o[:, :, perm]) and close(lse3, lse[:, :, perm])):
        return "Q permutation did not permute O"
    return None


def pin_key_shift(fwd, bwd):
    B, H, N, d = 1, 3, 8, 5
    q, k, v = rnd((B, H, N, d), 10), rnd((B, H, N, d), 11), rnd((B, H, N, d), 12)
    u = rnd((B, H, 1, d), 13)
    for causal in (False, True):
        o, lse = fwd(q, k, v, 0.8, causal)
        o2, lse2 = fwd(q, k + u, v, 0.8, causal)
        if not close(o, o2):
            return "key shift changed O"
        if not close(lse2 - lse, 0.8 * np.einsum("bhid,bhd->bhi", q, u[:, :, 0])):
            return "key shift: LSE did not move by scale q.u"
    return None


def pin_special_values(fwd, bwd):
    B, H, N, d = 1, 2, 10, 3
    q, k, v = rnd((B, H, N, d), 14), rnd((B, H, N, d), 15), rnd((B, H, N, d), 16)
    for causal in (False, True):
        o, _ = fwd(q, k, np.ones_like(v), 0.4, causal)
        if not close(o, np.ones_like(v)):
            return "V = 1 does not give O = 1"
        o, _ = fwd(q, k, v, 0.4, causal)
        if causal and not close(o[:, :, 0], v[:, :, 0]):
            return "causal row 0: O_0 != V_0"
    o, lse = fwd(q, k, v, 0.0, False)
    if not (close(o, np.broadcast_to(v.mean(2, keepdims=True), o.shape)) and close(lse, np.log(N) + 0 * lse)):
        return "scale 0 does not give mean(V), ln N"
    o, _ = fwd(q, k, v, 0.0, True)
    if not close(o, np.cumsum(v, 2) / np.arange(1, N + 1)[None, None, :, None]):
        return "scale 0, causal: not the prefix mean"
    return None


def pin_grad_identities(fwd, bwd):
    B, H, N, d = 2, 2, 11, 6
    q, k, v, dO = (rnd((B, H, N, d), s) for s in range(20, 24))
    for causal in (False, True):
        dq, dk, dv = bwd(q, k, v, dO, 0.45, causal)
        if not close(dk.sum(2), np.zeros((B, H, d)), 1e-9):
            return "sum_j dK_j != 0"
        if not close(dv.sum(2), dO.sum(2), 1e-9):
            return "sum_j dV_j != sum_i dO_i"
        if not close((q * dq).sum((2, 3)), (k * dk).sum((2, 3)), 1e-9):
            return "sum Q.dQ != sum K.dK"
    return None


def pin_finite_differences(fwd, bwd):
    h = 1e-6
    for (N, d, causal, seed) in ((1, 2, False, 30), (3, 4, False, 31), (3, 4, True, 32),
                                 (8, 8, False, 33), (8, 2, True, 34)):
        q, k, v, dO = (rnd((1, 1, N, d), seed + 10 * s) for s in range(4))
        sc = 0.7
        grads = bwd(q, k, v, dO, sc, causal)
        args = [q, k, v]
        for which in range(3):
            num = np.zeros_like(args[which])
            for idx in np.ndindex(args[which].shape):
                plus = [a.copy() for a in args]
                minus = [a.copy() for a in args]
                plus[which][idx] += h
                minus[which][idx] -= h
                lp = (fwd(*plus, sc, causal)[0] * dO).sum()
                lm = (fwd(*minus, sc, causal)[0] * dO).sum()
                num[idx] = (lp - lm) / (2 * h)
            g = grads[which]
            err = np.abs(g - num).max() / max(1.0, np.abs(num).max())
            if err > 1e-6:
                return f"finite differences: d{'QKV'[which]} N={N} d={d} causal={causal} err={err:.2e}"
    return None


def pin_torch_sdpa(fwd, bwd):
    import torch
    import torch.nn.functional as F
    for (B, H, N, d, causal, seed) in ((1, 2, 17, 8, False, 40), (2, 1, 13, 4, True, 41),
                                       (1, 1, 33, 16, True, 42)):
        q, k, v, dO = (rnd((B, H, N, d), seed + 100 * s) for s in range(4))
        sc = 1.0 / np.sqrt(d)
        tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
        to = F.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=sc)
        to.backward(torch.tensor(dO))
        o, _ = fwd(q, k, v, sc, causal)
        if not close(o, to.detach().numpy(), 1e-11):
            return f"forward differs from torch SDPA (N={N}, causal={causal})"
        dq, dk, dv = bwd(q, k, v, dO, sc, causal)
        for nm, a, b in (("dQ", dq, tq.grad), ("dK", dk, tk.grad), ("dV", dv, tv.grad)):
            if not close(a, b.numpy(), 1e-10):
                return f"{nm} differs from torch autograd (N={N}, causal={causal})"
    return None


PINS = [pin_golden, pin_n1, pin_identical_keys, pin_rows_sum_to_one, pin_permutations,
        pin_key_shift, pin_special_values, pin_grad_identities, pin_finite_differences,
        pin_torch_sdpa]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_c_oracle_passes(pin):
    msg = pin(c_fwd, c_bwd)
    assert msg is None, msg


# ---------------------------------------------------- planted mistakes

def _mutant(flaw):
    """NumPy restatement of attention with one deliberate mistake."""

    def scores(q, k, scale, causal):
        s = np.einsum("bhid,bhjd->bhij", q, k)
        if flaw != "no_scale":
            s = scale * s
        if causal:
            n = q.shape[2]
            keep = np.tril(np.ones((n, n), dtype=bool))
            if flaw == "mask_excludes_diag":
                keep = np.tril(np.ones((n, n), dtype=bool), -1)
                keep[0, 0] = True
            if flaw == "mask_transposed":
                keep = keep.T
            s = np.where(keep, s, -np.inf)
        return s

    def probs(q, k, scale, causal):
        s = scores(q, k, scale, causal)
        ax = -2 if flaw == "softmax_over_queries" else -1
        m = s.max(axis=ax, keepdims=True)
        e = np.exp(s - m)
        l = e.sum(axis=ax, keepdims=True)
        return e / l, m, l

    def fwd(q, k, v, scale, causal):
        p, m, l = probs(q, k, scale, causal)
        o = (np.swapaxes(p, -1, -2) if flaw == "p_transposed" else p) @ v
        if flaw == "v_index_shift":
            o = p @ np.roll(v, 1, axis=2)
        lse = np.log(l) if flaw == "lse_drops_max" else m + np.log(l)
        lse = lse[..., 0] if lse.shape[-1] == 1 else lse[..., 0, :]
        return o, lse

    def bwd(q, k, v, dO, scale, causal):
        p, _, _ = probs(q, k, scale, causal)
        dv = (p if flaw == "dv_untransposed" else np.swapaxes(p, -1, -2)) @ dO
        dp = dO @ np.swapaxes(v, -1, -2)
        D = (p * dp).sum(axis=-1, keepdims=True)
        if flaw == "ds_drops_D":
            ds = p * dp
        elif flaw == "ds_sign":
            ds = p * (D - dp)
        else:
            ds = p * (dp - D)
        dq = (1.0 if flaw == "dq_no_scale" else scale) * ds @ (v if flaw == "dq_uses_v" else k)
        dk = (1.0 if flaw == "dk_no_scale" else scale) * np.swapaxes(ds, -1, -2) @ q
        return dq, dk, dv

    return fwd, bwd


FLAWS = ["no_scale", "mask_excludes_diag", "mask_transposed", "softmax_over_queries",
         "p_transposed", "v_index_shift", "lse_drops_max", "dv_untransposed", "ds_drops_D",
         "ds_sign", "dq_no_scale", "dq_uses_v", "dk_no_scale"]


def test_numpy_restatement_passes():
    """The unmutated NumPy restatement passes too (so mutants fail for their flaw)."""
    def f(q, k, v, s, c):
        o, lse, _ = ref_numpy.np_fwd(q, k, v, s, c)
        return o, lse
    for pin in PINS:
        msg = pin(f, ref_numpy.np_bwd)
        assert msg is None, f"{pin.__name__}: {msg}"


@pytest.mark.parametrize("flaw", FLAWS)
def test_planted_mistakes_are_caught(flaw):
    fwd, bwd = _mutant(flaw)
    failures = []
    for pin in PINS:
        try:
            with np.errstate(all="ignore"):
                msg = pin(fwd, bwd)
        except Exception as e:  # a mutant may also crash a pin
            msg = f"raised {type(e).__name__}"
        if msg is not None:
            failures.append(pin.__name__)
    assert failures, f"planted mistake '{flaw}' slipped through every pin"


# ------------------------------------------------ cross-checks and helpers

@pytest.mark.parametrize("causal", [False, True])
def test_c_matches_numpy_restatement(causal):
    B, H, N, d = 2, 3, 37, 16
    q, k, v, dO = (rnd((B, H, N, d), 50 + s) for s in range(4))
    o, lse = c_fwd(q, k, v, 0.25, causal)
    o2, lse2, _ = ref_numpy.np_fwd(q, k, v, 0.25, causal)
    assert close(o, o2, 1e-12) and close(lse, lse2, 1e-12)
    for a, b in zip(c_bwd(q, k, v, dO, 0.25, causal), ref_numpy.np_bwd(q, k, v, dO, 0.25, causal)):
        assert close(a, b, 1e-11)


@pytest.mark.parametrize("causal", [False, True])
def test_sampled_rows_match_full(causal):
    B, H, N, d = 2, 2, 50, 8
    q, k, v, dO = (rnd((B, H, N, d), 60 + s) for s in range(4))
    o, lse = c_fwd(q, k, v, 0.3, causal)
    dq, _, _ = c_bwd(q, k, v, dO, 0.3, causal)
    sb = np.array([0, 3, 1, 2, 3, 0])
    sr = np.array([0, 49, 17, 1, 25, 48])
    os_, ls = oracle.ref_fwd_rows(q, k, v, 0.3, causal, sb, sr)
    dqs = oracle.ref_dq_rows(q, k, v, dO, 0.3, causal, sb, sr)
    of, lf, dqf = o.reshape(B * H, N, d), lse.reshape(B * H, N), dq.reshape(B * H, N, d)
    assert close(os_, of[sb, sr], 1e-13) and close(ls, lf[sb, sr], 1e-13)
    assert close(dqs, dqf[sb, sr], 1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_sampled_key_rows_match_full(causal):
    B, H, N, d = 1, 3, 45, 8
    q, k, v, dO = (rnd((B, H, N, d), 80 + s) for s in range(4))
    _, dk, dv = c_bwd(q, k, v, dO, 0.3, causal)
    for head in (0, 2):
        keys = np.array([44, 3, 20, 43, 0])
        dks, dvs = oracle.ref_dkdv_rows(q, k, v, dO, 0.3, causal, head, keys)
        assert close(dks, dk.reshape(B * H, N, d)[head, keys], 1e-12)
        assert close(dvs, dv.reshape(B * H, N, d)[head, keys], 1e-12)
    tail = np.arange(40, 45)
    dks, dvs = oracle.ref_dkdv_rows(q, k, v, dO, 0.3, causal, 1, tail)
    assert close(dks, dk.reshape(B * H, N, d)[1, tail], 1e-12)
    assert close(dvs, dv.reshape(B * H, N, d)[1, tail], 1e-12)


def test_thread_count_does_not_change_forward():
    q, k, v = (rnd((1, 2, 64, 8), 70 + s) for s in range(3))
    o1, l1 = oracle.ref_fwd(q, k, v, 0.3, True, nthreads=1)
    o8, l8 = oracle.ref_fwd(q, k, v, 0.3, True, nthreads=8)
    assert np.array_equal(o1, o8) and np.array_equal(l1, l8)


def test_bf16_inputs_widen_exactly():
    import torch
    t = torch.randn(1, 1, 5, 4).to(torch.bfloat16)
    o, _ = oracle.ref_fwd(t, t, t, 0.5, False)
    o2, _ = oracle.ref_fwd(t.float().numpy().astype(np.float64), t.float().numpy().astype(np.float64),
                           t.float().numpy().astype(np.float64), 0.5, False)
    assert np.array_equal(o, o2)


def test_bad_arguments_rejected():
    q = np.zeros((1, 1, 4, 2))
    with pytest.raises(RuntimeError):
        oracle.ref_fwd_rows(q, q, q, 1.0, False, [0], [4])
    with pytest.raises(RuntimeError):
        oracle.ref_fwd_rows(q, q, q, 1.0, False, [1], [0])


def test_score_matrix_bytes_matches_pages_example():
    from io_aware_exact_23_b200.inputs import score_matrix_bytes
    with open(os.path.join(GOLDEN, "score_matrix_bytes.json")) as f:
        g = json.load(f)
    for c in g["cases"]:
        assert score_matrix_bytes(c["B"], c["H"], c["N"], c["elem_bytes"]) == c["bytes"]
