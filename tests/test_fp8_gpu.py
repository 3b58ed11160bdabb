"""GPU parity of the e4m3 forward (fa_fwd_fp8, through the C ABI) against the
fp64 oracle of the dequantised inputs (``oracle.fp8``).

Gate, element by element, on the error before the output's final rounding to
bf16 (the distance from O_ref to the reals that round to the returned value):

    pre_ic <= bound_ic + slack_i

* bound = ``oracle.fp8.p_rounding_bound``: rounding P to e4m3 before the PV
  product (relative 2^-4, absolute 2^-10), pinned on the CPU;
* slack_i: the fp32 arithmetic of S.  S_ij sums d exact products of e4m3 values
  in fp32, so |dS_ij| <= g * scale * sum_c |q_ic k_jc| with g = d u / (1 - d u),
  u = 2^-24 (any summation order).  A shift of every S_ij by at most e moves
  each weight P_ij / l_i by a factor within exp(+-2e), hence O_i by at most
  expm1(2 e_i) * max_jc |V_jc| with e_i = max_j of that bound.
LSE is gated at 1e-3 plus e_i.  The inputs follow ``make_fp8_inputs`` (the
bf16 workloads' fp32 draws, per-head descale = max|x| / 448).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from oracle import fp8
from io_aware_exact_23_b200 import binding as fa
from io_aware_exact_23_b200.inputs import C3, Workload, make_fp8_inputs

from gpu_helpers import rounding_interval

pytestmark = pytest.mark.gpu

U32 = 2.0 ** -24


def run_fp8(w: Workload):
    t = make_fp8_inputs(w, device="cuda")
    o = torch.full((w.B, w.H, w.N, w.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((w.B, w.H, w.N), float("nan"), dtype=torch.float32, device="cuda")
    fa.fa_fwd_fp8(t["q"], t["k"], t["v"], t["dq"], t["dk"], t["dv"], o, lse, w.scale, w.causal)
    st, info = fa.fa_device_status(info=True)
    assert st == 0, f"device status {st} {info}"
    return t, o, lse


def s_slack(q, k, scale, causal):
    """Per-row bound e_i on the fp32 error of S (fp64 arrays [N, d] of one head)."""
    d = q.shape[1]
    g = d * U32 / (1.0 - d * U32)
    a = scale * (np.abs(q) @ np.abs(k).T)
    if causal:
        a = np.where(np.tril(np.ones(a.shape, dtype=bool)), a, 0.0)
    return g * a.max(axis=1)


def check_heads(w: Workload, heads=None):
    t, o, lse = run_fp8(w)
    BH = w.B * w.H
    heads = range(BH) if heads is None else heads
    o_all = o.reshape(BH, w.N, w.d)
    lse_all = lse.reshape(BH, w.N).double().cpu().numpy()
    worst = 0.0
    for bh in heads:
        b, h = divmod(bh, w.H)
        sl = {nm: t[nm][b:b + 1, h:h + 1] for nm in ("q", "k", "v")}
        ds = {nm: t["d" + nm][b:b + 1, h:h + 1] for nm in ("q", "k", "v")}
        qd, kd, vd = (fp8.dequantize(sl[nm], ds[nm]) for nm in ("q", "k", "v"))
        o_ref, l_ref = oracle.ref_fwd(qd, kd, vd, w.scale, w.causal)
        bound = fp8.p_rounding_bound(qd, kd, vd, w.scale, w.causal)[0, 0]
        e = s_slack(qd[0, 0], kd[0, 0], w.scale, w.causal)
        slack = np.expm1(2.0 * e)[:, None] * np.abs(vd).max()
        oh = o_all[bh]
        got = oh.double().cpu().numpy()
        assert np.isfinite(got).all(), f"{w.name} head {bh}: non-finite O"
        lo, hi = rounding_interval(oh)
        ref = o_ref[0, 0]
        pre = np.maximum(np.maximum(lo - ref, ref - hi), 0.0)
        excess = pre - (bound + slack)
        assert excess.max() <= 0.0, (f"{w.name} head {bh}: O error before rounding exceeds the bound by "
                                     f"{excess.max():.3e} (max pre {pre.max():.3e})")
        el = np.abs(lse_all[bh] - l_ref[0, 0])
        assert (el <= 1e-3 + e).all(), f"{w.name} head {bh}: max|LSE - LSE_ref| = {el.max():.3e}"
        worst = max(worst, float((pre / np.maximum(bound + slack, 1e-300)).max()))
    return worst


EDGE = [(n, c) for c in (False, True) for n in (1, 17, 128, 129, 255, 257, 300)]


@pytest.mark.parametrize("N,causal", EDGE, ids=lambda x: str(x))
def test_fp8_ragged_and_edge_lengths(N, causal):
    check_heads(Workload(f"fp8_edge_n{N}", 1, 2, N, 128, causal, seed=N))


@pytest.mark.parametrize("causal", [False, True])
def test_fp8_multi_head_ragged(causal):
    check_heads(Workload("fp8_mh", 2, 3, 1000, 128, causal, seed=7))


@pytest.mark.parametrize("causal", [False, True])
def test_fp8_stress_x8(causal):
    """Q, K x 8 before quantisation: near one-hot rows, frequent max updates."""
    check_heads(Workload("fp8_stress", 1, 2, 768, 128, causal, qk_mult=8.0, seed=3))


def test_fp8_bench_workload_two_heads():
    """B=2, H=32, N=4096, d=128, causal: whole heads 0 and 63 of the full launch."""
    check_heads(Workload("fp8_" + C3.name, C3.B, C3.H, C3.N, C3.d, C3.causal), heads=[0, C3.B * C3.H - 1])


@pytest.mark.parametrize("mult", [1.0, 8.0])
def test_fp8_sweep_point(mult):
    """Sweep point B=4, H=16, N=4096, non-causal (and its x8 twin): two whole heads."""
    w = Workload("fp8_sweep_b4h16n4096d128", 4, 16, 4096, 128, False, qk_mult=mult)
    check_heads(w, heads=[5, 63])


def test_fp8_row0_causal_is_v0():
    """Causal row 0 attends to key 0 only: O_0 = V_0 * descale_v (P = 1 is exact in e4m3)."""
    w = Workload("fp8_row0", 1, 4, 512, 128, True, seed=11)
    t, o, _ = run_fp8(w)
    v0 = fp8.dequantize(t["v"], t["dv"])[:, :, 0]
    got = o[:, :, 0].double().cpu().numpy()
    lo, hi = rounding_interval(o[:, :, 0])
    assert ((v0 >= lo - 1e-12) & (v0 <= hi + 1e-12)).all()
    assert np.isfinite(got).all()
