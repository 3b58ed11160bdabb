"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle.

Every input comes from the seeded generator (io_aware_exact_23_b200.inputs);
every expected value comes from ``oracle``.  Small shapes are compared element
by element over whole tensors; the full-size workloads are compared at sampled
(head, row) positions the oracle computes one by one (O, LSE, dQ rows; dK, dV
rows of one head: the whole head up to N = 4096 -- 1024 in the sweep -- else
key tiles 0, middle and last), plus gradient identities that hold at any size:  sum_j dK_j = 0,  sum_j dV_j = sum_i dO_i  and
sum_i Q_i.dQ_i = sum_j K_j.dK_j.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_23_b200 import inputs as I
from io_aware_exact_23_b200.inputs import Workload, make_inputs

from gpu_helpers import (TOL_GRAD_REL, TOL_LSE, TOL_O, full_check, gate_o, gpu_backward, gpu_forward, max_err,
                         record_parity, sample_rows, to64)

pytestmark = pytest.mark.gpu


# ------------------------------------------------------------ small, full
def test_tiny_config_full():
    full_check(I.TINY)


EDGE = [(n, d, c) for d in (64, 128) for c in (False, True) for n in (1, 17, 128, 129, 255, 257, 300)]


@pytest.mark.parametrize("N,d,causal", EDGE, ids=lambda x: str(x))
def test_ragged_and_edge_lengths_full(N, d, causal):
    full_check(Workload(f"edge_n{N}", 1, 2, N, d, causal, seed=N))


@pytest.mark.parametrize("d,causal", [(64, False), (64, True), (128, False), (128, True)])
def test_multi_head_ragged_full(d, causal):
    full_check(Workload("mh", 2, 3, 1000, d, causal, seed=7))


@pytest.mark.parametrize("d,causal", [(64, False), (64, True), (128, False), (128, True)])
def test_stress_x8_full(d, causal):
    """Q, K x 8: logits with std ~ 64 (near one-hot rows, frequent max updates)."""
    full_check(Workload("stress", 1, 2, 768, d, causal, qk_mult=8.0, seed=3))


@pytest.mark.parametrize("w", [I.TINY, Workload("plain_c", 2, 3, 1000, 128, True, seed=5),
                               Workload("plain_n", 1, 4, 640, 64, False, seed=6)], ids=lambda w: w.name)
def test_plain_entry_points_full(w):
    """fa_fwd / fa_bwd without the O residual (D from the bf16 O) on N(0,1) inputs."""
    full_check(w, residual=False)


def test_residual_tracks_fp32_output():
    """o + o_lo is much closer to O_ref than o alone."""
    w = Workload("resid", 1, 4, 512, 128, False, seed=15)
    t = make_inputs(w, device="cuda")
    o, lse, o_lo = gpu_forward(t, w.scale, False, residual=True)
    o2, lse2 = gpu_forward(t, w.scale, False)
    assert torch.equal(o, o2) and torch.equal(lse, lse2)
    # the residual is what rounding dropped: it lies inside the rounding half-gap of o
    from gpu_helpers import rounding_interval
    lo, hi = rounding_interval(o)
    tot = to64(o) + to64(o_lo)
    assert ((tot >= lo - 1e-12) & (tot <= hi + 1e-12)).all()
    o_ref, _ = oracle.ref_fwd(t["q"], t["k"], t["v"], w.scale, False)
    assert max_err(tot, o_ref) <= max_err(to64(o), o_ref)


# ------------------------------------------------------------ exactness
def test_causal_row0_is_v0_exactly():
    w = Workload("row0", 2, 4, 512, 128, True, seed=11)
    t = make_inputs(w, device="cuda")
    o, _ = gpu_forward(t, w.scale, True)
    assert torch.equal(o[:, :, 0], t["v"][:, :, 0])


@pytest.mark.parametrize("d,causal", [(64, False), (128, True)])
def test_forward_is_deterministic(d, causal):
    """Bit-identical output over repeated launches that fill every SM.  The
    forward overwrites a tile's P in TMEM with its next S, ordered only by the
    tensor pipe's in-order execution: a hazard there would show up as run-to-run
    differences."""
    w = Workload("det", 2, 16, 2048, d, causal, seed=12)
    t = make_inputs(w, device="cuda")
    o1, l1 = gpu_forward(t, w.scale, causal)
    for _ in range(12):
        o2, l2 = gpu_forward(t, w.scale, causal)
        assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_outputs_stay_inside_their_buffers():
    """Guard bands of NaN around every output are left untouched."""
    from io_aware_exact_23_b200 import binding as fa
    w = Workload("guard", 1, 3, 300, 128, True, seed=13)
    t = make_inputs(w, device="cuda")
    n = w.elems()
    G = 4096  # guard elements on each side (16-byte multiples keep alignment)

    def guarded(numel, dtype):
        buf = torch.full((numel + 2 * G,), float("nan"), dtype=dtype, device="cuda")
        return buf, buf[G:G + numel]

    ob, o = guarded(n, torch.bfloat16)
    lb, lse = guarded(w.B * w.H * w.N, torch.float32)
    o, lse = o.view(t["q"].shape), lse.view(w.B, w.H, w.N)
    fa.fa_fwd(t["q"], t["k"], t["v"], o, lse, w.scale, True)
    grads = [guarded(n, torch.bfloat16) for _ in range(3)]
    ws = torch.zeros(fa.fa_bwd_workspace_bytes(w.B, w.H, w.N, w.d), dtype=torch.uint8, device="cuda")
    fa.fa_bwd(t["q"], t["k"], t["v"], o, t["do"], lse, *(g[1].view(t["q"].shape) for g in grads), w.scale,
              True, ws)
    assert fa.fa_device_status() == 0
    for buf in [ob, lb] + [g[0] for g in grads]:
        assert torch.isnan(buf[:G].float()).all() and torch.isnan(buf[-G:].float()).all()
    for x in [o, lse] + [g[1] for g in grads]:
        assert torch.isfinite(x.float()).all()


def test_argument_error_touches_nothing():
    from io_aware_exact_23_b200 import binding as fa
    L = fa.lib()
    q = torch.randn(1, 1, 256, 64, device="cuda").to(torch.bfloat16)
    o = torch.full_like(q, 7.0)
    lse = torch.full((1, 1, 256), 7.0, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    assert L.fa_fwd(q.data_ptr(), q.data_ptr(), q.data_ptr(), o.data_ptr(), lse.data_ptr(),
                    1, 1, 256, 96, 0.1, 0, s) == 2
    assert L.fa_fwd(q.data_ptr(), q.data_ptr(), q.data_ptr(), o.data_ptr(), lse.data_ptr(),
                    1, 1, 256, 64, float("nan"), 0, s) == 1
    assert L.fa_fwd(q.data_ptr() + 2, q.data_ptr(), q.data_ptr(), o.data_ptr(), lse.data_ptr(),
                    1, 1, 256, 64, 0.1, 0, s) == 3
    torch.cuda.synchronize()
    assert (o == 7.0).all() and (lse == 7.0).all()
    assert fa.fa_device_status() == 0


def test_non_default_stream():
    w = Workload("stream", 1, 4, 640, 64, True, seed=14)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        t = make_inputs(w, device="cuda")
        o, lse = gpu_forward(t, w.scale, True)
    o_ref, l_ref = oracle.ref_fwd(t["q"], t["k"], t["v"], w.scale, True)
    assert max_err(to64(o), o_ref) <= TOL_O and max_err(to64(lse), l_ref) <= TOL_LSE


# ------------------------------------------------------ full-size workloads
def key_tile_rows(N: int) -> np.ndarray:
    """Key rows of three 128-row key tiles: tile 0, a middle tile and the last
    (ragged) tile.  When causal, tile 0 accumulates every query tile and the
    last tile only the diagonal one; non-causal, each sees every query tile."""
    nt = (N + 127) // 128
    tiles = sorted({0, nt // 2, nt - 1})
    return np.concatenate([np.arange(t * 128, min(N, (t + 1) * 128)) for t in tiles])


def check_sampled(w: Workload, n_rows=192, dkdv_full_head_max_n=4096):
    t = make_inputs(w, device="cuda")
    o, lse, o_lo = gpu_forward(t, w.scale, w.causal, residual=True)
    dq, dk, dv = gpu_backward(t, o, lse, w.scale, w.causal, o_lo=o_lo)
    BH, N, d = w.B * w.H, w.N, w.d
    sb, sr = sample_rows(BH, N, n_rows, seed=w.N + d)
    o_ref, l_ref = oracle.ref_fwd_rows(t["q"], t["k"], t["v"], w.scale, w.causal, sb, sr)
    sbt, srt = torch.as_tensor(sb, device="cuda"), torch.as_tensor(sr, device="cuda")
    o_s = o.reshape(BH, N, d)[sbt, srt]
    olo_s = o_lo.reshape(BH, N, d)[sbt, srt]
    lf = to64(lse).reshape(BH, N)
    eo, epre, eres = gate_o(w, o_s, o_ref, olo_s, w.name + " (sampled)")
    el = max_err(lf[sb, sr], l_ref)
    assert el <= TOL_LSE, f"{w.name}: sampled max|LSE-LSE_ref| = {el:.3e}"
    # dQ at the same rows; the gate's scale is the oracle's max over the sampled rows
    dq_ref = oracle.ref_dq_rows(t["q"], t["k"], t["v"], t["do"], w.scale, w.causal, sb, sr)
    dqf = to64(dq).reshape(BH, N, d)
    e = max_err(dqf[sb, sr], dq_ref)
    rel = {"dq": e / np.abs(dq_ref).max()}
    assert e <= TOL_GRAD_REL * np.abs(dq_ref).max(), f"{w.name}: sampled dQ err {e:.3e}"
    # dK, dV rows of one head, element by element: the whole head when it is
    # affordable, else key tiles 0, middle and last (see key_tile_rows).
    dkf, dvf = to64(dk).reshape(BH, N, d), to64(dv).reshape(BH, N, d)
    head = int(np.random.default_rng(w.N).integers(0, BH))
    keys = np.arange(N) if N <= dkdv_full_head_max_n else key_tile_rows(N)
    rk, rv = oracle.ref_dkdv_rows(t["q"], t["k"], t["v"], t["do"], w.scale, w.causal, head, keys)
    for nm, g, r in (("dK", dkf[head, keys], rk), ("dV", dvf[head, keys], rv)):
        e = max_err(g, r)
        rel[nm.lower()] = e / np.abs(r).max()
        assert e <= TOL_GRAD_REL * np.abs(r).max(), f"{w.name}: {nm} err {e:.3e} vs {np.abs(r).max():.3e}"
    record_parity(w, "sampled", strict=eo, pre_rounding=epre, residual=eres, lse=el, grads_rel=rel,
                  dkdv_keys=int(len(keys)), head=head)
    # identities over every head, in fp64 on the GPU outputs (extra checks)
    q64 = t["q"].double()
    k64 = t["k"].double()
    dk64, dv64, dq64 = dk.double(), dv.double(), dq.double()
    s_dk = dk64.sum(2)
    bound_dk = TOL_GRAD_REL * dk64.abs().amax(dim=(2, 3), keepdim=False) * np.sqrt(N)
    assert (s_dk.abs().amax(dim=2) <= bound_dk + 1e-6).all(), f"{w.name}: sum_j dK_j != 0"
    s_dv = dv64.sum(2) - t["do"].double().sum(2)
    bound_dv = TOL_GRAD_REL * dv64.abs().amax(dim=(2, 3)) * np.sqrt(N)
    assert (s_dv.abs().amax(dim=2) <= bound_dv + 1e-6).all(), f"{w.name}: sum_j dV_j != sum_i dO_i"
    lhs = (q64 * dq64).sum((2, 3))
    rhs = (k64 * dk64).sum((2, 3))
    mag = (q64.abs() * dq64.abs()).sum((2, 3)) + (k64.abs() * dk64.abs()).sum((2, 3))
    assert ((lhs - rhs).abs() <= TOL_GRAD_REL * mag).all(), f"{w.name}: sum Q.dQ != sum K.dK"
    return {"o": eo, "lse": el}


@pytest.mark.parametrize("w", [I.C2, I.C3], ids=lambda w: w.name)
def test_full_size_configs(w):
    check_sampled(w)


@pytest.mark.slow
def test_long_context_config():
    check_sampled(I.C4, n_rows=96)


SWEEP = I.sweep()


@pytest.mark.parametrize("w", SWEEP, ids=lambda w: w.name)
def test_sweep_point(w):
    check_sampled(w, n_rows=64, dkdv_full_head_max_n=1024)


@pytest.mark.slow
def test_very_long_sequence_sampled():
    """B=1, H=1, N=262144, d=128, causal: 64x the long-context workload's tokens
    per head.  O, LSE and dQ at sampled rows (first, tile edges, middle, last)
    against the oracle, dK / dV element by element on the last key tile (whose
    query statistics are cheap to get at this N), and the gradient identities
    over the whole head."""
    w = Workload("very_long_b1h1n262144d128_causal", 1, 1, 262144, 128, True, seed=17)
    t = make_inputs(w, device="cuda")
    o, lse, o_lo = gpu_forward(t, w.scale, True, residual=True)
    dq, dk, dv = gpu_backward(t, o, lse, w.scale, True, o_lo=o_lo)
    N, d = w.N, w.d
    sb, sr = sample_rows(1, N, 24, seed=N)
    o_ref, l_ref = oracle.ref_fwd_rows(t["q"], t["k"], t["v"], w.scale, True, sb, sr)
    of, lf = to64(o).reshape(N, d), to64(lse).reshape(N)
    assert max_err(of[sr], o_ref) <= TOL_O
    assert max_err(lf[sr], l_ref) <= TOL_LSE
    dq_ref = oracle.ref_dq_rows(t["q"], t["k"], t["v"], t["do"], w.scale, True, sb, sr)
    assert max_err(to64(dq).reshape(N, d)[sr], dq_ref) <= TOL_GRAD_REL * np.abs(dq_ref).max()
    keys = np.arange(N - 128, N)
    rk, rv = oracle.ref_dkdv_rows(t["q"], t["k"], t["v"], t["do"], w.scale, True, 0, keys)
    for g, r in ((to64(dk).reshape(N, d)[keys], rk), (to64(dv).reshape(N, d)[keys], rv)):
        assert max_err(g, r) <= TOL_GRAD_REL * np.abs(r).max()
    dk64, dv64, dq64 = dk.double(), dv.double(), dq.double()
    assert (dk64.sum(2).abs().amax() <= TOL_GRAD_REL * dk64.abs().amax() * np.sqrt(N) + 1e-6).all()
    s_dv = (dv64.sum(2) - t["do"].double().sum(2)).abs().amax()
    assert s_dv <= TOL_GRAD_REL * dv64.abs().amax() * np.sqrt(N) + 1e-6
    lhs = (t["q"].double() * dq64).sum()
    rhs = (t["k"].double() * dk64).sum()
    mag = (t["q"].double().abs() * dq64.abs()).sum() + (t["k"].double().abs() * dk64.abs()).sum()
    assert (lhs - rhs).abs() <= TOL_GRAD_REL * mag
