"""ctypes binding of libfa_vanilla.so, the standard-attention baseline.

Argument marshalling only, as in ``binding.py``: the C entry points declared in
``include/fa_vanilla.h`` do the work (cuBLAS GEMMs and the library's own row
softmax kernels).  Raises at import if ``libfa_vanilla.so`` was not built.
"""
from __future__ import annotations

import ctypes
import os

import torch

from .binding import FA_OK, FaError, _check, _stream_handle

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfa_vanilla.so")
_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise ImportError(f"{_LIB_PATH} not found: build it with `python -m io_aware_exact_23_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        L.fa_vanilla_workspace_bytes.argtypes = [i, i, i, i]
        L.fa_vanilla_workspace_bytes.restype = sz
        L.fa_vanilla_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, vp, sz, vp]
        L.fa_vanilla_fwd.restype = i
        L.fa_vanilla_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, vp, sz, vp]
        L.fa_vanilla_bwd.restype = i
        _lib = L
    return _lib


lib()


def workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return int(lib().fa_vanilla_workspace_bytes(B, H, N, d))


def fwd(q, k, v, o, lse, scale: float, causal: bool, workspace, stream=None) -> None:
    """Standard attention forward; ``workspace`` (uint8, CUDA) keeps S and P."""
    B, H, N, d = q.shape
    for nm, t in (("q", q), ("k", k), ("v", v), ("o", o)):
        _check(t, nm, torch.bfloat16, (B, H, N, d))
    _check(lse, "lse", torch.float32, (B, H, N))
    _check(workspace, "workspace", torch.uint8)
    rc = lib().fa_vanilla_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H, N, d,
                              float(scale), int(bool(causal)), workspace.data_ptr(), workspace.numel(),
                              _stream_handle(stream))
    if rc != FA_OK:
        raise FaError(rc, "fa_vanilla_fwd")


def bwd(q, k, v, o, dO, lse, dq, dk, dv, scale: float, causal: bool, workspace, stream=None) -> None:
    """Standard attention backward from the P that ``fwd`` left in ``workspace``."""
    B, H, N, d = q.shape
    for nm, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dO", dO), ("dq", dq), ("dk", dk), ("dv", dv)):
        _check(t, nm, torch.bfloat16, (B, H, N, d))
    _check(lse, "lse", torch.float32, (B, H, N))
    _check(workspace, "workspace", torch.uint8)
    rc = lib().fa_vanilla_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dO.data_ptr(), lse.data_ptr(),
                              dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, N, d, float(scale),
                              int(bool(causal)), workspace.data_ptr(), workspace.numel(), _stream_handle(stream))
    if rc != FA_OK:
        raise FaError(rc, "fa_vanilla_bwd")
