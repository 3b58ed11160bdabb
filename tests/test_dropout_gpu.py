"""GPU parity of fused dropout: the mask (bit-exact against the oracle's
generator), the forward and backward with dropout (the same gates as without),
rate 0 reproducing the dropout-free kernels bit for bit, and masks that change
with the offset."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_23_b200 import binding as fa
from io_aware_exact_23_b200.inputs import Workload, make_inputs

from gpu_helpers import TOL_LSE, TOL_O, check_grads, max_err, o_errors, to64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,H,N,rate,seed,offset", [
    (1, 3, 200, 0.1, 0, 0), (2, 2, 130, 0.5, 0xFEDCBA9876543210, 7), (1, 1, 17, 0.9, 12345, 1 << 31),
    (1, 2, 64, 0.0, 3, 3), (1, 1, 33, 0.003, 5, 0)])
def test_mask_is_bit_exact(B, H, N, rate, seed, offset):
    mask = torch.full((B, H, N, N), 7, dtype=torch.uint8, device="cuda")
    fa.fa_dropout_mask(B, H, N, rate, seed, offset, mask)
    torch.cuda.synchronize()
    ref = oracle.dropout_mask(B * H, N, seed, offset, rate).reshape(B, H, N, N)
    assert np.array_equal(mask.cpu().numpy(), ref)


def run_dropout(t, w, rate, seed, offset, residual=True):
    q, k, v, dO = t["q"], t["k"], t["v"], t["do"]
    B, H, N, d = q.shape
    o = torch.full_like(q, float("nan"))
    o_lo = torch.full_like(q, float("nan")) if residual else None
    lse = torch.full((B, H, N), float("nan"), dtype=torch.float32, device=q.device)
    fa.fa_fwd_dropout(q, k, v, o, lse, w.scale, w.causal, rate, seed, offset, o_lo=o_lo)
    ws = torch.full((fa.fa_bwd_workspace_bytes(B, H, N, d),), 0xFF, dtype=torch.uint8, device=q.device)
    dq, dk, dv = (torch.full_like(q, float("nan")) for _ in range(3))
    fa.fa_bwd_dropout(q, k, v, o, dO, lse, dq, dk, dv, w.scale, w.causal, rate, seed, ws, offset=offset, o_lo=o_lo)
    st, info = fa.fa_device_status(info=True)
    assert st == 0, (st, info)
    return o, lse, o_lo, dq, dk, dv


CASES = [Workload(f"drop_n{N}_d{d}_c{int(c)}", 1, 2, N, d, c, seed=5)
         for N in (129, 300) for d in (64, 128) for c in (False, True)] + [
    Workload("drop_b2h2n1000d128c", 2, 2, 1000, 128, True, seed=6)]


@pytest.mark.parametrize("rate", [0.1, 0.5])
@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_dropout_matches_oracle(w, rate):
    seed, offset = 0x9E3779B97F4A7C15, 11
    t = make_inputs(w, device="cuda")
    o, lse, o_lo, dq, dk, dv = run_dropout(t, w, rate, seed, offset)
    o_ref, lse_ref = oracle.ref_fwd_dropout(t["q"], t["k"], t["v"], w.scale, w.causal, rate, seed, offset)
    # With dropout O is no convex combination of V rows: kept entries are scaled by
    # 1/(1 - rate), so |O| can pass 4, where half a bf16 spacing alone exceeds 1e-2.
    # O is gated before that final rounding (as for the x8 stress inputs): the
    # rounding interval of the returned value, and o + o_lo, must be within 1e-2.
    strict, pre, res = o_errors(o, o_ref, o_lo)
    assert pre <= TOL_O and res <= TOL_O, (strict, pre, res)
    assert max_err(to64(lse), lse_ref) <= TOL_LSE
    rq, rk, rv = oracle.ref_bwd_dropout(t["q"], t["k"], t["v"], t["do"], w.scale, w.causal, rate, seed, offset)
    check_grads({"dq": to64(dq), "dk": to64(dk), "dv": to64(dv)}, {"dq": rq, "dk": rk, "dv": rv}, w.name)


@pytest.mark.parametrize("d,causal,rate", [(64, False, 0.0), (128, True, 0.0), (128, False, 0.003)])
def test_rate_zero_is_the_plain_kernel(d, causal, rate):
    """Rate 0, or any rate below 1/256 (the rate's step: T = 0, every key kept,
    scale 1), reproduces the dropout-free kernels."""
    w = Workload("drop0", 2, 3, 700, d, causal, seed=8)
    t = make_inputs(w, device="cuda")
    o, lse, _, dq, dk, dv = run_dropout(t, w, rate, 1, 0, residual=False)
    o2 = torch.empty_like(o)
    lse2 = torch.empty_like(lse)
    fa.fa_fwd(t["q"], t["k"], t["v"], o2, lse2, w.scale, causal)
    assert torch.equal(o, o2) and torch.equal(lse, lse2)
    ws = torch.empty(fa.fa_bwd_workspace_bytes(*t["q"].shape), dtype=torch.uint8, device="cuda")
    dq2, dk2, dv2 = (torch.empty_like(o) for _ in range(3))
    fa.fa_bwd(t["q"], t["k"], t["v"], o2, t["do"], lse2, dq2, dk2, dv2, w.scale, causal, ws)
    torch.cuda.synchronize()
    assert torch.equal(dk, dk2) and torch.equal(dv, dv2)
    # dQ is summed over key tiles in arrival order: equal up to that order.
    assert max_err(to64(dq), to64(dq2)) <= 1e-2 * float(dq2.abs().max())


def test_offset_changes_the_mask_and_seed_reproduces_it():
    w = Workload("drop_off", 1, 2, 256, 64, False, seed=9)
    t = make_inputs(w, device="cuda")
    outs = []
    for offset in (0, 0, 1):
        o = torch.empty_like(t["q"])
        lse = torch.empty(t["q"].shape[:3], dtype=torch.float32, device="cuda")
        fa.fa_fwd_dropout(t["q"], t["k"], t["v"], o, lse, w.scale, False, 0.3, 42, offset)
        outs.append(o)
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1])
    assert not torch.equal(outs[0], outs[2])


def test_dropout_full_size_workload():
    """The bench's workload (B=2, H=32, N=4096, d=128, causal) with dropout 0.1 on the GPU;
    two whole heads (every element of O, LSE, dQ, dK, dV) against the oracle."""
    from io_aware_exact_23_b200.inputs import C3 as w
    rate, seed, offset = 0.1, 0x5EED, 3
    t = make_inputs(w, device="cuda")
    o, lse, o_lo, dq, dk, dv = run_dropout(t, w, rate, seed, offset)
    for b, h in ((0, 0), (1, 21)):
        sl = {nm: x[b:b + 1, h:h + 1] for nm, x in t.items()}
        head0 = b * w.H + h
        o_ref, lse_ref = oracle.ref_fwd_dropout(sl["q"], sl["k"], sl["v"], w.scale, True, rate, seed, offset,
                                                head0=head0)
        strict, pre, res = o_errors(o[b:b + 1, h:h + 1], o_ref, o_lo[b:b + 1, h:h + 1])
        assert pre <= TOL_O and res <= TOL_O, (b, h, strict, pre, res)
        assert max_err(to64(lse[b:b + 1, h:h + 1]), lse_ref) <= TOL_LSE
        rq, rk, rv = oracle.ref_bwd_dropout(sl["q"], sl["k"], sl["v"], sl["do"], w.scale, True, rate, seed, offset,
                                            head0=head0)
        check_grads({"dq": to64(dq[b:b + 1, h:h + 1]), "dk": to64(dk[b:b + 1, h:h + 1]),
                     "dv": to64(dv[b:b + 1, h:h + 1])}, {"dq": rq, "dk": rk, "dv": rv}, f"C3 head {head0}")
