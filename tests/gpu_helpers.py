"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI
and compare it with the fp64 oracle.

Tolerances (bf16 inputs, fp32 accumulation), element by element:
  max |O - O_ref|     <= 1e-2
  max |LSE - LSE_ref| <= 1e-3
  max |dX - dX_ref|   <= 2e-2 * max |dX_ref|   for dX in dQ, dK, dV separately
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from io_aware_exact_23_b200 import binding as fa
from io_aware_exact_23_b200.inputs import Workload, make_inputs

TOL_O = 1e-2
TOL_LSE = 1e-3
TOL_GRAD_REL = 2e-2


def gpu_forward(t, scale, causal):
    q, k, v = t["q"], t["k"], t["v"]
    B, H, N, d = q.shape
    o = torch.full_like(q, float("nan"))
    lse = torch.full((B, H, N), float("nan"), dtype=torch.float32, device=q.device)
    fa.fa_fwd(q, k, v, o, lse, scale, causal)
    st, info = fa.fa_device_status(info=True)
    assert st == 0, f"device status {st} {info}"
    return o, lse


def gpu_backward(t, o, lse, scale, causal):
    q, k, v, dO = t["q"], t["k"], t["v"], t["do"]
    B, H, N, d = q.shape
    ws = torch.full((fa.fa_bwd_workspace_bytes(B, H, N, d),), 0xFF, dtype=torch.uint8, device=q.device)
    dq, dk, dv = (torch.full_like(q, float("nan")) for _ in range(3))
    fa.fa_bwd(q, k, v, o, dO, lse, dq, dk, dv, scale, causal, ws)
    st, info = fa.fa_device_status(info=True)
    assert st == 0, f"device status {st} {info}"
    return dq, dk, dv


def to64(x):
    return x.detach().to("cpu", torch.float64).numpy()


def max_err(a, b):
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, (a.shape, b.shape)
    if a.size == 0:
        return 0.0
    assert np.isfinite(a).all(), "non-finite GPU output"
    return float(np.abs(a - b).max())


# Below this magnitude the relative gate becomes absolute (2e-2 x 1e-3 = 2e-5):
# at N = 1 the exact dQ and dK are identically zero.
GRAD_SCALE_FLOOR = 1e-3


def check_grads(got: dict, ref: dict, label=""):
    for nm in ("dq", "dk", "dv"):
        g, r = got[nm], ref[nm]
        scale = max(float(np.abs(r).max()), GRAD_SCALE_FLOOR)
        err = max_err(g, r)
        assert err <= TOL_GRAD_REL * scale, f"{label} {nm}: max err {err:.3e} > {TOL_GRAD_REL} x {scale:.3e}"


def full_check(w: Workload, device="cuda", check_bwd=True, nthreads=0):
    """Full-tensor comparison (small shapes): every element of O, LSE, dQ, dK, dV."""
    t = make_inputs(w, device=device)
    o, lse = gpu_forward(t, w.scale, w.causal)
    o_ref, lse_ref = oracle.ref_fwd(t["q"], t["k"], t["v"], w.scale, w.causal, nthreads=nthreads)
    eo, el = max_err(to64(o), o_ref), max_err(to64(lse), lse_ref)
    assert eo <= TOL_O, f"{w.name}: max|O - O_ref| = {eo:.3e}"
    assert el <= TOL_LSE, f"{w.name}: max|LSE - LSE_ref| = {el:.3e}"
    out = {"o": eo, "lse": el}
    if check_bwd:
        dq, dk, dv = gpu_backward(t, o, lse, w.scale, w.causal)
        rq, rk, rv = oracle.ref_bwd(t["q"], t["k"], t["v"], t["do"], w.scale, w.causal, nthreads=nthreads)
        check_grads({"dq": to64(dq), "dk": to64(dk), "dv": to64(dv)}, {"dq": rq, "dk": rk, "dv": rv}, w.name)
        for nm, g, r in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
            out[nm] = max_err(to64(g), r) / max(float(np.abs(r).max()), 1e-30)
    return out


def sample_rows(BH, N, n, seed=0):
    """Seeded (head, row) samples that always include the first and last rows and tile edges."""
    rng = np.random.default_rng(seed)
    bh = list(rng.integers(0, BH, size=n))
    rows = list(rng.integers(0, N, size=n))
    for r in {0, N - 1, min(127, N - 1), min(128, N - 1), N // 2}:
        bh.append(int(rng.integers(0, BH)))
        rows.append(r)
    return np.array(bh), np.array(rows)
