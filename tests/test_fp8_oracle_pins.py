"""Pins of the FP8 (e4m3) forward's reference and error bound (``oracle/fp8.py``), on the CPU.

* The e4m3 decoder, written from the format's bit layout, against torch's
  float8_e4m3fn conversion for all 256 codes, and the format's closed-form
  landmarks (448, 2^-6, 2^-9).
* The input recipe: every dequantised input is within e4m3's rounding error of
  the fp32 draw it came from.
* The reference: attention of the dequantised inputs equals torch's fp64
  scaled_dot_product_attention on them.
* The bound on rounding P to e4m3: a simulation of that rounding (torch's
  e4m3 conversion, at the scales a running max can leave) stays within it on
  N(0,1) and x8 inputs, causal or not; and it is not loose by a factor 2 (the
  bound with half the relative error fails on some case).
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

from io_aware_exact_23_b200.inputs import Workload, make_fp8_inputs
from oracle import fp8


def test_decoder_matches_torch_for_every_code():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    want = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = fp8.e4m3_values()
    assert np.array_equal(np.isnan(got), np.isnan(want))
    ok = ~np.isnan(want)
    assert np.array_equal(got[ok], want[ok])


def test_decoder_landmarks():
    t = fp8.e4m3_values()
    finite = t[~np.isnan(t)]
    assert finite.max() == 448.0 and finite.min() == -448.0
    assert t[0x08] == 2.0 ** -6 and t[0x01] == 2.0 ** -9 and t[0x00] == 0.0 and t[0x80] == 0.0
    pos = t[:0x7F]
    assert np.all(np.diff(pos) > 0)  # codes 0x00..0x7E increase strictly
    assert np.isnan(t[0x7F]) and np.isnan(t[0xFF])


@pytest.mark.parametrize("qk_mult", [1.0, 8.0])
def test_inputs_are_within_rounding_of_the_draws(qk_mult):
    w = Workload("fp8_in", 2, 3, 96, 64, False, qk_mult=qk_mult, seed=4)
    t = make_fp8_inputs(w)
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed)
    for nm in ("q", "k", "v"):
        x = torch.randn((w.B, w.H, w.N, w.d), generator=g, dtype=torch.float32).double().numpy()
        if nm in ("q", "k"):
            x = x * qk_mult
        deq = fp8.dequantize(t[nm], t["d" + nm])
        s = t["d" + nm].double().numpy()[:, :, None, None]
        tol = np.maximum(fp8.REL_ERR * np.abs(x), fp8.ABS_ERR * s) * (1 + 1e-6)
        assert np.all(np.abs(deq - x) <= tol), nm
        assert np.allclose(np.abs(deq).max(axis=(2, 3)), 448.0 * s[:, :, 0, 0], rtol=1e-6)


@pytest.mark.parametrize("causal", [False, True])
def test_reference_is_attention_of_the_dequantised_inputs(causal):
    w = Workload("fp8_ref", 1, 2, 80, 32, causal, seed=5)
    t = make_fp8_inputs(w)
    o, lse = fp8.ref_fwd_fp8(t["q"], t["k"], t["v"], t["dq"], t["dk"], t["dv"], w.scale, causal)
    q, k, v = (torch.from_numpy(fp8.dequantize(t[n], t["d" + n])) for n in ("q", "k", "v"))
    want = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=causal, scale=w.scale)
    assert np.allclose(o, want.numpy(), rtol=0, atol=1e-12)
    s = w.scale * torch.einsum("bhid,bhjd->bhij", q, k)
    if causal:
        s = s.masked_fill(~torch.ones(w.N, w.N, dtype=torch.bool).tril(), -math.inf)
    assert np.allclose(lse, torch.logsumexp(s, dim=-1).numpy(), rtol=0, atol=1e-12)


def simulate_fp8_pv(q, k, v, scale, causal, shift_log2, rel_err=None):
    """O with P rounded to e4m3 (torch's conversion), P taken at 2^shift times its
    value relative to the row max (a running max below the true one)."""
    B, H, N, d = q.shape
    out = np.empty_like(q)
    for b in range(B):
        for h in range(H):
            s = scale * (q[b, h] @ k[b, h].T)
            if causal:
                s = np.where(np.tril(np.ones((N, N), dtype=bool)), s, -np.inf)
            p = np.exp(s - s.max(axis=1, keepdims=True)) * (2.0 ** shift_log2[b, h][:, None])
            p8 = torch.from_numpy(p).to(torch.float8_e4m3fn).to(torch.float64).numpy()
            out[b, h] = (p8 @ v[b, h]) / p.sum(axis=1, keepdims=True)
    return out


CASES = [(1, 2, 128, 64, False, 1.0), (1, 2, 128, 64, True, 1.0), (1, 2, 200, 128, True, 8.0),
         (2, 1, 96, 64, False, 8.0), (1, 1, 300, 32, True, 1.0)]


@pytest.mark.parametrize("B,H,N,d,causal,mult", CASES)
def test_bound_holds_for_p_rounded_to_e4m3(B, H, N, d, causal, mult):
    w = Workload("fp8_bound", B, H, N, d, causal, qk_mult=mult, seed=N + d)
    t = make_fp8_inputs(w)
    q, k, v = (fp8.dequantize(t[n], t["d" + n]) for n in ("q", "k", "v"))
    o_ref, _ = fp8.ref_fwd_fp8(t["q"], t["k"], t["v"], t["dq"], t["dk"], t["dv"], w.scale, causal)
    bound = fp8.p_rounding_bound(q, k, v, w.scale, causal)
    rng = np.random.default_rng(N)
    for shifts in (np.zeros((B, H, N)), rng.uniform(0.0, 8.0, size=(B, H, N))):
        o = simulate_fp8_pv(q, k, v, w.scale, causal, shifts)
        assert np.all(np.abs(o - o_ref) <= bound * (1 + 1e-9) + 1e-12)


def test_bound_is_not_loose_by_two():
    """Halving the relative rounding error in the bound is caught on one of the cases."""
    caught = False
    for B, H, N, d, causal, mult in CASES:
        w = Workload("fp8_tight", B, H, N, d, causal, qk_mult=mult, seed=N + d)
        t = make_fp8_inputs(w)
        q, k, v = (fp8.dequantize(t[n], t["d" + n]) for n in ("q", "k", "v"))
        o_ref, _ = fp8.ref_fwd_fp8(t["q"], t["k"], t["v"], t["dq"], t["dk"], t["dv"], w.scale, causal)
        half = fp8.p_rounding_bound(q, k, v, w.scale, causal) / 2
        o = simulate_fp8_pv(q, k, v, w.scale, causal, np.zeros((B, H, N)))
        caught |= bool(np.any(np.abs(o - o_ref) > half))
    assert caught
