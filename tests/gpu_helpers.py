"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI
and compare it with the fp64 oracle.

Tolerances (bf16 inputs, fp32 accumulation), element by element:
  max |O - O_ref|     <= 1e-2
  max |LSE - LSE_ref| <= 1e-3
  max |dX - dX_ref|   <= 2e-2 * max |dX_ref|   for dX in dQ, dK, dV separately

O is a bf16 output: once |O| >= 2 half of a bf16 spacing is 2^-7 or more, and
at |O| >= 4 it is 2^-6 > 1e-2, so rounding the output alone can exceed 1e-2.
For the x8 stress inputs (where |O| reaches 4 in near one-hot rows) the O gate
is therefore applied to the result before that final rounding: the distance
from O_ref to the set of reals that round to the returned bf16 value must be
<= 1e-2, and so must |(o + o_lo) - O_ref|, where o_lo is the rounding residual
the forward returns.  Every other workload is gated on the strict form.
"""
from __future__ import annotations

import json
import os

import numpy as np
import torch

import oracle
from io_aware_exact_23_b200 import binding as fa
from io_aware_exact_23_b200.inputs import Workload, make_inputs

TOL_O = 1e-2
TOL_LSE = 1e-3
TOL_GRAD_REL = 2e-2


def gpu_forward(t, scale, causal, residual=False):
    """(o, lse) or, with residual=True, (o, lse, o_lo)."""
    q, k, v = t["q"], t["k"], t["v"]
    B, H, N, d = q.shape
    o = torch.full_like(q, float("nan"))
    o_lo = torch.full_like(q, float("nan")) if residual else None
    lse = torch.full((B, H, N), float("nan"), dtype=torch.float32, device=q.device)
    fa.fa_fwd(q, k, v, o, lse, scale, causal, o_lo=o_lo)
    st, info = fa.fa_device_status(info=True)
    assert st == 0, f"device status {st} {info}"
    return (o, lse, o_lo) if residual else (o, lse)


def gpu_backward(t, o, lse, scale, causal, o_lo=None):
    q, k, v, dO = t["q"], t["k"], t["v"], t["do"]
    B, H, N, d = q.shape
    ws = torch.full((fa.fa_bwd_workspace_bytes(B, H, N, d),), 0xFF, dtype=torch.uint8, device=q.device)
    dq, dk, dv = (torch.full_like(q, float("nan")) for _ in range(3))
    fa.fa_bwd(q, k, v, o, dO, lse, dq, dk, dv, scale, causal, ws, o_lo=o_lo)
    st, info = fa.fa_device_status(info=True)
    assert st == 0, f"device status {st} {info}"
    return dq, dk, dv


def rounding_interval(x: torch.Tensor):
    """For bf16 values x: (lo, hi) fp64 bounds of the reals that round (RNE) to x."""
    xs = x.detach().contiguous()
    bits = xs.view(torch.int16).to(torch.int32)
    sign = bits < 0
    mag = bits & 0x7FFF
    up = (mag + 1).to(torch.int16).view(torch.bfloat16).double().abs()
    down = (mag - 1).clamp(min=0).to(torch.int16).view(torch.bfloat16).double().abs()
    a = xs.double().abs()
    hi_mag = a + (up - a) / 2
    lo_mag = torch.where(mag == 0, -hi_mag, a - (a - down) / 2)
    lo = torch.where(sign, -hi_mag, lo_mag)
    hi = torch.where(sign, -lo_mag, hi_mag)
    return lo.cpu().numpy(), hi.cpu().numpy()


def o_errors(o: torch.Tensor, o_ref, o_lo: torch.Tensor | None = None):
    """Strict, pre-rounding (interval) and residual-based max errors of O."""
    strict = max_err(to64(o), o_ref)
    lo, hi = rounding_interval(o)
    pre = float(np.maximum(np.maximum(lo - o_ref, o_ref - hi), 0.0).max()) if o_ref.size else 0.0
    res = max_err(to64(o) + to64(o_lo), o_ref) if o_lo is not None else None
    return strict, pre, res


def gate_o(w: Workload, o, o_ref, o_lo=None, label=""):
    strict, pre, res = o_errors(o, o_ref, o_lo)
    if w.qk_mult == 1.0:
        assert strict <= TOL_O, f"{label}: max|O - O_ref| = {strict:.3e}"
    else:
        assert pre <= TOL_O, f"{label}: O error before output rounding {pre:.3e} (strict {strict:.3e})"
        if res is not None:
            assert res <= TOL_O, f"{label}: max|o + o_lo - O_ref| = {res:.3e} (strict {strict:.3e})"
    return strict, pre, res


def record_parity(w: Workload, kind: str, **errs):
    """Append one JSON line of measured errors to the file named by the
    FA_PARITY_LOG environment variable (no-op when it is unset).  The strict
    max|O - O_ref| is recorded beside the pre-rounding and residual errors the
    stress gate uses, flagged when it exceeds 1e-2."""
    path = os.environ.get("FA_PARITY_LOG")
    if not path:
        return
    rec = {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal,
           "qk_mult": w.qk_mult, "kind": kind}
    rec.update({k: (None if v is None else (float(v) if np.isscalar(v) else v)) for k, v in errs.items()})
    strict = errs.get("strict")
    rec["strict_over_1e-2"] = bool(strict is not None and strict > TOL_O)
    with open(path, "a") as f:
        f.write(json.dumps(rec) + "\n")


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


def full_check(w: Workload, device="cuda", check_bwd=True, nthreads=0, residual=True):
    """Full-tensor comparison (small shapes): every element of O, LSE, dQ, dK, dV."""
    t = make_inputs(w, device=device)
    if residual:
        o, lse, o_lo = gpu_forward(t, w.scale, w.causal, residual=True)
    else:
        (o, lse), o_lo = gpu_forward(t, w.scale, w.causal), None
    o_ref, lse_ref = oracle.ref_fwd(t["q"], t["k"], t["v"], w.scale, w.causal, nthreads=nthreads)
    eo, epre, eres = gate_o(w, o, o_ref, o_lo, w.name)
    el = max_err(to64(lse), lse_ref)
    assert el <= TOL_LSE, f"{w.name}: max|LSE - LSE_ref| = {el:.3e}"
    out = {"o": eo, "lse": el}
    if check_bwd:
        dq, dk, dv = gpu_backward(t, o, lse, w.scale, w.causal, o_lo=o_lo)
        rq, rk, rv = oracle.ref_bwd(t["q"], t["k"], t["v"], t["do"], w.scale, w.causal, nthreads=nthreads)
        check_grads({"dq": to64(dq), "dk": to64(dk), "dv": to64(dv)}, {"dq": rq, "dk": rk, "dv": rv}, w.name)
        for nm, g, r in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
            out[nm] = max_err(to64(g), r) / max(float(np.abs(r).max()), 1e-30)
    record_parity(w, "full", strict=eo, pre_rounding=epre, residual=eres, lse=el,
                  grads_rel={k: out[k] for k in ("dq", "dk", "dv") if k in out})
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
