"""fa_bwd_noalloc: the backward pass for callers that cannot allocate device
memory (code running inside its own allocator or memory pool, under a fixed
real-time memory budget, or where a host framework owns all device memory).
Its scratch is a fixed static array inside libfa.so instead of a caller
workspace.  These tests check, through the C ABI, that two calls in a row give
the same gradients as fa_bwd within the parity tolerance, and that a shape
needing more scratch than the array holds is refused before any launch.

This file is named so that pytest collects it last."""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

from io_aware_exact_23_b200 import binding as fa
from io_aware_exact_23_b200.inputs import Workload, make_inputs

pytestmark = pytest.mark.gpu

TOL_GRAD_REL = 2e-2  # max|dX - dX_ref| <= 2e-2 * max|dX_ref|, as in the parity tests


def _grads_with_workspace(t, o, lse, w):
    B, H, N, d = t["q"].shape
    ws = torch.empty(fa.fa_bwd_workspace_bytes(B, H, N, d), dtype=torch.uint8, device="cuda")
    out = [torch.empty_like(t["q"]) for _ in range(3)]
    fa.fa_bwd(t["q"], t["k"], t["v"], o, t["do"], lse, *out, w.scale, w.causal, ws)
    assert fa.fa_device_status() == 0
    return out


def _grads_noalloc(t, o, lse, w):
    B, H, N, d = t["q"].shape
    out = [torch.full_like(t["q"], float("nan")) for _ in range(3)]
    L = fa.lib()
    rc = L.fa_bwd_noalloc(t["q"].data_ptr(), t["k"].data_ptr(), t["v"].data_ptr(), o.data_ptr(),
                          t["do"].data_ptr(), lse.data_ptr(), out[0].data_ptr(), out[1].data_ptr(),
                          out[2].data_ptr(), B, H, N, d, ctypes.c_float(w.scale), int(w.causal),
                          torch.cuda.current_stream().cuda_stream)
    assert rc == 0, L.fa_status_string(rc)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("w", [Workload("noalloc_c", 2, 4, 1000, 128, True, seed=21),
                               Workload("noalloc_n", 1, 3, 700, 64, False, seed=22)], ids=lambda w: w.name)
def test_noalloc_matches_workspace_backward_on_two_calls(w):
    assert fa.fa_bwd_workspace_bytes(w.B, w.H, w.N, w.d) <= fa.NOALLOC_SCRATCH_BYTES
    t = make_inputs(w, device="cuda")
    B, H, N, d = t["q"].shape
    o = torch.empty_like(t["q"])
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    fa.fa_fwd(t["q"], t["k"], t["v"], o, lse, w.scale, w.causal)
    ref = _grads_with_workspace(t, o, lse, w)
    for call in range(2):  # the static scratch keeps the previous call's contents
        got = _grads_noalloc(t, o, lse, w)
        for nm, g, r in zip(("dq", "dk", "dv"), got, ref):
            g64, r64 = g.double().cpu().numpy(), r.double().cpu().numpy()
            assert np.isfinite(g64).all(), f"call {call}: {nm} not finite"
            err = np.abs(g64 - r64).max()
            assert err <= TOL_GRAD_REL * max(np.abs(r64).max(), 1e-3), f"call {call}: {nm} err {err:.3e}"


def test_noalloc_refuses_shapes_beyond_its_scratch():
    L = fa.lib()
    B, H, N, d = 2, 32, 4096, 128  # needs ~136 MB of scratch
    assert fa.fa_bwd_workspace_bytes(B, H, N, d) > fa.NOALLOC_SCRATCH_BYTES
    p = ctypes.c_void_p(4096)  # never dereferenced: the size check comes first
    rc = L.fa_bwd_noalloc(p, p, p, p, p, p, p, p, p, B, H, N, d, ctypes.c_float(0.088), 1, None)
    assert rc == 4, L.fa_status_string(rc)
