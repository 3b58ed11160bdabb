"""Host-side tests of the standard-attention baseline's C ABI (no GPU needed):
libfa_vanilla.so loads, exports what include/fa_vanilla.h declares, sizes its
O(N^2) workspace as documented and rejects bad arguments before any launch."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa_vanilla.h")


@pytest.fixture(scope="module")
def vlib():
    from io_aware_exact_23_b200 import build
    build.build()
    build.build_vanilla()
    from io_aware_exact_23_b200 import vanilla
    return vanilla.lib()


def declared_functions():
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", src)))


def test_exports(vlib):
    names = declared_functions()
    assert names == ["fa_vanilla_bwd", "fa_vanilla_fwd", "fa_vanilla_workspace_bytes"]
    for nm in names:
        assert hasattr(vlib, nm)


def test_workspace_is_six_bytes_per_score(vlib):
    for B, H, N, d in [(1, 1, 1, 64), (2, 32, 4096, 128), (1, 2, 300, 128)]:
        want = 6 * B * H * N * N
        assert vlib.fa_vanilla_workspace_bytes(B, H, N, d) == (want + 255) // 256 * 256
    assert vlib.fa_vanilla_workspace_bytes(1, 1, 256, 96) == 0
    assert vlib.fa_vanilla_workspace_bytes(0, 1, 256, 64) == 0


P = ctypes.c_void_p(4096)
BAD = ctypes.c_void_p(4097)


def fwd(vlib, *, q=P, ws=P, ws_bytes=1 << 40, B=1, H=2, N=256, d=64, scale=0.125, causal=0):
    return vlib.fa_vanilla_fwd(q, P, P, P, P, B, H, N, d, scale, causal, ws, ws_bytes, None)


def bwd(vlib, *, dq=P, ws=P, ws_bytes=1 << 40, N=256, d=64, scale=0.125):
    return vlib.fa_vanilla_bwd(P, P, P, P, P, P, dq, P, P, 1, 2, N, d, scale, 0, ws, ws_bytes, None)


def test_argument_errors(vlib):
    assert fwd(vlib, d=96) == 2                  # unsupported head dim
    assert fwd(vlib, N=0) == 1                   # invalid shape
    assert fwd(vlib, scale=float("nan")) == 1    # non-finite scale
    assert fwd(vlib, causal=2) == 1
    assert fwd(vlib, q=ctypes.c_void_p(0)) == 1  # null pointer
    assert fwd(vlib, q=BAD) == 3                 # misaligned
    assert fwd(vlib, ws_bytes=100) == 4          # workspace too small
    assert bwd(vlib, d=96) == 2
    assert bwd(vlib, dq=BAD) == 3
    assert bwd(vlib, ws=ctypes.c_void_p(0)) == 1
    assert bwd(vlib, ws_bytes=100) == 4


def test_no_device_is_reported(vlib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert fwd(vlib) == 5 and bwd(vlib) == 5
