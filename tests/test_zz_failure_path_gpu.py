"""The device-side failure path on the GPU, without a fault.

Every pipeline wait in the kernels is bounded: when its time limit passes it
records FA_ERR_DEVICE_TIMEOUT with the kernel, wait tag, block and launch
sequence number in the library's status word, and the kernel returns.
``fa_selftest_timeout`` launches one thread whose wait can never complete (a
barrier nothing arrives on), so that path runs for real.  Checked: the status
and the record come back to the host, reading the status clears it, and the
context stays usable (a forward right after it is correct).
"""
from __future__ import annotations

import time

import pytest
import torch

import oracle
from io_aware_exact_23_b200 import binding as fa
from io_aware_exact_23_b200.inputs import Workload, make_inputs

from gpu_helpers import TOL_LSE, TOL_O, gpu_forward, max_err, to64

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_the_context_survives():
    assert fa.fa_device_status() == 0
    t0 = time.monotonic()
    fa.fa_selftest_timeout()
    st, info = fa.fa_device_status(info=True)  # synchronises: the wait gives up after 1 s
    waited = time.monotonic() - t0
    assert st == 7, f"status {st}"  # FA_ERR_DEVICE_TIMEOUT
    kernel, tag, block, seq = info
    assert (kernel, tag, block) == (5, 1, 0) and seq > 0, info
    assert waited >= 0.9, f"gave up after {waited:.3f} s"
    assert fa.fa_device_status() == 0  # read once, then cleared
    w = Workload("after_timeout", 1, 2, 300, 128, True, seed=31)
    t = make_inputs(w, device="cuda")
    o, lse = gpu_forward(t, w.scale, True)
    o_ref, l_ref = oracle.ref_fwd(t["q"], t["k"], t["v"], w.scale, True)
    assert max_err(to64(o), o_ref) <= TOL_O and max_err(to64(lse), l_ref) <= TOL_LSE
    torch.cuda.synchronize()
