"""GPU parity of the standard-attention baseline (libfa_vanilla.so) against the
fp64 oracle, with the same gates as the IO-aware kernels (N(0,1) workloads),
and a cross-check that the baseline and the IO-aware path agree."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_23_b200.inputs import TINY, Workload, make_inputs

from gpu_helpers import TOL_LSE, TOL_O, check_grads, gpu_backward, gpu_forward, max_err, to64

pytestmark = pytest.mark.gpu


def vanilla_step(t, scale, causal):
    from io_aware_exact_23_b200 import vanilla
    q, k, v, dO = t["q"], t["k"], t["v"], t["do"]
    B, H, N, d = q.shape
    ws = torch.full((vanilla.workspace_bytes(B, H, N, d),), 0xFF, dtype=torch.uint8, device=q.device)
    o = torch.full_like(q, float("nan"))
    lse = torch.full((B, H, N), float("nan"), dtype=torch.float32, device=q.device)
    vanilla.fwd(q, k, v, o, lse, scale, causal, ws)
    dq, dk, dv = (torch.full_like(q, float("nan")) for _ in range(3))
    vanilla.bwd(q, k, v, o, dO, lse, dq, dk, dv, scale, causal, ws)
    torch.cuda.synchronize()
    return o, lse, dq, dk, dv


CASES = [TINY] + [Workload(f"van_n{N}_d{d}_c{int(c)}", 1, 3, N, d, c, seed=7)
                  for N in (1, 17, 129, 300) for d in (64, 128) for c in (False, True)] + [
    Workload("van_b2h4n1024d128c", 2, 4, 1024, 128, True, seed=3)]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_vanilla_matches_oracle(w):
    t = make_inputs(w, device="cuda")
    o, lse, dq, dk, dv = vanilla_step(t, w.scale, w.causal)
    o_ref, lse_ref = oracle.ref_fwd(t["q"], t["k"], t["v"], w.scale, w.causal)
    assert max_err(to64(o), o_ref) <= TOL_O
    assert max_err(to64(lse), lse_ref) <= TOL_LSE
    rq, rk, rv = oracle.ref_bwd(t["q"], t["k"], t["v"], t["do"], w.scale, w.causal)
    check_grads({"dq": to64(dq), "dk": to64(dk), "dv": to64(dv)}, {"dq": rq, "dk": rk, "dv": rv}, w.name)


def test_vanilla_and_io_aware_agree():
    """Both GPU paths on one input: outputs within the sum of their oracle gates."""
    w = Workload("van_vs_fa", 2, 4, 768, 128, True, seed=21)
    t = make_inputs(w, device="cuda")
    o, lse, dq, dk, dv = vanilla_step(t, w.scale, w.causal)
    o2, lse2 = gpu_forward(t, w.scale, w.causal)
    dq2, dk2, dv2 = gpu_backward(t, o2, lse2, w.scale, w.causal)
    assert max_err(to64(o), to64(o2)) <= 2 * TOL_O
    assert max_err(to64(lse), to64(lse2)) <= 2 * TOL_LSE
    for a, b in ((dq, dq2), (dk, dk2), (dv, dv2)):
        assert max_err(to64(a), to64(b)) <= 4e-2 * float(np.abs(to64(b)).max())
