"""ctypes binding of libfa.so: argument marshalling only.

Every function here checks tensor dtypes/shapes/devices, turns torch tensors
into raw device pointers and the current CUDA stream into a handle, and calls
the C entry point of the same name declared in ``include/fa.h``.  All
arithmetic happens in the CUDA kernels.  If ``libfa.so`` is missing this module
raises at import: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfa.so")

FA_OK = 0
STATUS_NAMES = {
    0: "FA_OK", 1: "FA_ERR_INVALID_ARG", 2: "FA_ERR_UNSUPPORTED", 3: "FA_ERR_MISALIGNED",
    4: "FA_ERR_WORKSPACE", 5: "FA_ERR_NO_DEVICE", 6: "FA_ERR_CUDA", 7: "FA_ERR_DEVICE_TIMEOUT",
    8: "FA_ERR_DEVICE_INTERNAL",
}


class FaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {lib().fa_status_string(code).decode()} ({code})")


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libfa.so (raises ImportError if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise ImportError(
                f"{_LIB_PATH} not found: build it with `python -m io_aware_exact_23_b200.build` "
                "(the attention path has no CPU fallback)")
        L = ctypes.CDLL(_LIB_PATH)
        vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        L.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, vp]
        L.fa_fwd.restype = i
        L.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, vp, sz, vp]
        L.fa_bwd.restype = i
        L.fa_fwd_residual.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, vp]
        L.fa_fwd_residual.restype = i
        L.fa_bwd_ex.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, vp, sz, vp,
                                ctypes.POINTER(vp)]
        L.fa_bwd_ex.restype = i
        u64, u32 = ctypes.c_ulonglong, ctypes.c_uint
        L.fa_fwd_fp8.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, vp]
        L.fa_fwd_fp8.restype = i
        L.fa_fwd_dropout.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, f, u64, u32, vp]
        L.fa_fwd_dropout.restype = i
        L.fa_bwd_dropout.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, f, u64, u32, vp, sz,
                                     vp]
        L.fa_bwd_dropout.restype = i
        L.fa_dropout_mask.argtypes = [i, i, i, f, u64, u32, vp, vp]
        L.fa_dropout_mask.restype = i
        L.fa_bwd_deterministic.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, vp, sz, vp]
        L.fa_bwd_deterministic.restype = i
        L.fa_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, vp]
        L.fa_bwd_noalloc.restype = i
        L.fa_bwd_workspace_bytes.argtypes = [i, i, i, i]
        L.fa_bwd_workspace_bytes.restype = sz
        L.fa_status_string.argtypes = [i]
        L.fa_status_string.restype = ctypes.c_char_p
        L.fa_device_status.argtypes = [vp]
        L.fa_device_status.restype = i
        L.fa_device_status_info.argtypes = [vp, ctypes.POINTER(ctypes.c_int)]
        L.fa_device_status_info.restype = i
        L.fa_selftest_timeout.argtypes = [vp]
        L.fa_selftest_timeout.restype = i
        L.fa_noalloc_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_int)]
        L.fa_noalloc_device_status.restype = i
        L.fa_noalloc_selftest_timeout.argtypes = [vp]
        L.fa_noalloc_selftest_timeout.restype = i
        L.fa_version.argtypes = []
        L.fa_version.restype = i
        _lib = L
    return _lib


lib()  # fail at import when the extension is missing


def _stream_handle(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _check(t: torch.Tensor, name: str, dtype, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def fa_fwd(q, k, v, o, lse, scale: float, causal: bool, stream=None, o_lo=None) -> None:
    """O and LSE into the preallocated ``o`` [B,H,N,d] bf16 and ``lse`` [B,H,N] fp32.

    ``o_lo``: optional bf16 tensor shaped like ``o`` that receives O's rounding
    residual (``fa_fwd_residual``), for an exact backward ``D``.
    """
    B, H, N, d = q.shape
    for nm, t in (("q", q), ("k", k), ("v", v), ("o", o)):
        _check(t, nm, torch.bfloat16, (B, H, N, d))
    _check(lse, "lse", torch.float32, (B, H, N))
    if o_lo is None:
        rc = lib().fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                          B, H, N, d, float(scale), int(bool(causal)), _stream_handle(stream))
    else:
        _check(o_lo, "o_lo", torch.bfloat16, (B, H, N, d))
        rc = lib().fa_fwd_residual(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), o_lo.data_ptr(),
                                   lse.data_ptr(), B, H, N, d, float(scale), int(bool(causal)),
                                   _stream_handle(stream))
    if rc != FA_OK:
        raise FaError(rc, "fa_fwd")


def fa_fwd_fp8(q8, k8, v8, descale_q, descale_k, descale_v, o, lse, scale: float, causal: bool,
               stream=None) -> None:
    """FP8 forward: ``q8``, ``k8``, ``v8`` are uint8 e4m3 codes [B,H,N,d] (d = 128),
    ``descale_*`` fp32 [B,H] per-head factors (inputs = code * descale); O into the
    bf16 ``o`` [B,H,N,d] and LSE into the fp32 ``lse`` [B,H,N]."""
    B, H, N, d = q8.shape
    for nm, t in (("q8", q8), ("k8", k8), ("v8", v8)):
        _check(t, nm, torch.uint8, (B, H, N, d))
    for nm, t in (("descale_q", descale_q), ("descale_k", descale_k), ("descale_v", descale_v)):
        _check(t, nm, torch.float32, (B, H))
    _check(o, "o", torch.bfloat16, (B, H, N, d))
    _check(lse, "lse", torch.float32, (B, H, N))
    rc = lib().fa_fwd_fp8(q8.data_ptr(), k8.data_ptr(), v8.data_ptr(), descale_q.data_ptr(), descale_k.data_ptr(),
                          descale_v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H, N, d, float(scale),
                          int(bool(causal)), _stream_handle(stream))
    if rc != FA_OK:
        raise FaError(rc, "fa_fwd_fp8")


def fa_bwd_workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return int(lib().fa_bwd_workspace_bytes(B, H, N, d))


def fa_bwd(q, k, v, o, dO, lse, dq, dk, dv, scale: float, causal: bool, workspace, stream=None,
           events=None, o_lo=None) -> None:
    """dQ, dK, dV into preallocated bf16 tensors; ``workspace`` is a uint8 CUDA tensor.

    ``o_lo``: the residual from ``fa_fwd(..., o_lo=...)`` (optional).
    ``events``: optional sequence of four ``torch.cuda.Event(enable_timing=True)``
    recorded around the preprocess, main and dQ-conversion kernels.
    """
    B, H, N, d = q.shape
    for nm, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dO", dO), ("dq", dq), ("dk", dk), ("dv", dv)):
        _check(t, nm, torch.bfloat16, (B, H, N, d))
    _check(lse, "lse", torch.float32, (B, H, N))
    _check(workspace, "workspace", torch.uint8)
    if events is None and o_lo is None:
        rc = lib().fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dO.data_ptr(), lse.data_ptr(),
                          dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, N, d, float(scale),
                          int(bool(causal)), workspace.data_ptr(), workspace.numel(), _stream_handle(stream))
    else:
        handles = None
        if events is not None:
            if len(events) != 4:
                raise ValueError("events must hold four torch.cuda.Event objects")
            for ev in events:
                if ev.cuda_event == 0:  # torch creates the CUDA event lazily, on first record
                    ev.record()
            handles = (ctypes.c_void_p * 4)(*[ev.cuda_event for ev in events])
        if o_lo is not None:
            _check(o_lo, "o_lo", torch.bfloat16, (B, H, N, d))
        rc = lib().fa_bwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                             None if o_lo is None else o_lo.data_ptr(), dO.data_ptr(), lse.data_ptr(),
                             dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, N, d, float(scale),
                             int(bool(causal)), workspace.data_ptr(), workspace.numel(), _stream_handle(stream),
                             handles)
    if rc != FA_OK:
        raise FaError(rc, "fa_bwd")


def fa_bwd_deterministic(q, k, v, o, dO, lse, dq, dk, dv, scale: float, causal: bool, workspace, stream=None,
                         o_lo=None) -> None:
    """``fa_bwd`` with dQ summed over key tiles in a fixed order: the same bits on
    every call (``fa_bwd_deterministic``); dK and dV are ``fa_bwd``'s."""
    B, H, N, d = q.shape
    for nm, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dO", dO), ("dq", dq), ("dk", dk), ("dv", dv)):
        _check(t, nm, torch.bfloat16, (B, H, N, d))
    _check(lse, "lse", torch.float32, (B, H, N))
    _check(workspace, "workspace", torch.uint8)
    if o_lo is not None:
        _check(o_lo, "o_lo", torch.bfloat16, (B, H, N, d))
    rc = lib().fa_bwd_deterministic(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                    o_lo.data_ptr() if o_lo is not None else None, dO.data_ptr(), lse.data_ptr(),
                                    dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, N, d, float(scale),
                                    int(bool(causal)), workspace.data_ptr(), workspace.numel(),
                                    _stream_handle(stream))
    if rc != FA_OK:
        raise FaError(rc, "fa_bwd_deterministic")


NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024  # FA_NOALLOC_SCRATCH_BYTES in include/fa.h


def fa_bwd_noalloc(q, k, v, o, dO, lse, dq, dk, dv, scale: float, causal: bool, stream=None) -> None:
    """``fa_bwd`` for callers that cannot allocate device memory: no workspace
    argument; the scratch is a fixed static array inside libfa.so (shapes that
    need more than NOALLOC_SCRATCH_BYTES are refused).  Calls that overlap on
    the GPU share that array and race; the first call on a device does a
    one-time set-up and should come before any stream capture."""
    B, H, N, d = q.shape
    for nm, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dO", dO), ("dq", dq), ("dk", dk), ("dv", dv)):
        _check(t, nm, torch.bfloat16, (B, H, N, d))
    _check(lse, "lse", torch.float32, (B, H, N))
    rc = lib().fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dO.data_ptr(),
                              lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, N, d,
                              float(scale), int(bool(causal)), _stream_handle(stream))
    if rc != FA_OK:
        raise FaError(rc, "fa_bwd_noalloc")


def fa_noalloc_device_status(stream=None, info: bool = False):
    """Synchronise the stream and return (and clear) fa_bwd_noalloc's own status code."""
    buf = (ctypes.c_int * 4)()
    rc = lib().fa_noalloc_device_status(_stream_handle(stream), buf)
    return (rc, list(buf)) if info else rc


def fa_noalloc_selftest_timeout(stream=None) -> None:
    """The failure-path self-test aimed at fa_bwd_noalloc's status word."""
    rc = lib().fa_noalloc_selftest_timeout(_stream_handle(stream))
    if rc != FA_OK:
        raise FaError(rc, "fa_noalloc_selftest_timeout")


def fa_device_status(stream=None, info: bool = False):
    """Synchronise the stream and return (and clear) the device status code."""
    buf = (ctypes.c_int * 4)()
    rc = lib().fa_device_status_info(_stream_handle(stream), buf)
    return (rc, list(buf)) if info else rc


def fa_selftest_timeout(stream=None) -> None:
    """Launch the failure-path self-test: a wait that gives up after its 1 s limit
    and records FA_ERR_DEVICE_TIMEOUT, which ``fa_device_status`` then returns."""
    rc = lib().fa_selftest_timeout(_stream_handle(stream))
    if rc != FA_OK:
        raise FaError(rc, "fa_selftest_timeout")


class Attention:
    """Allocating convenience wrapper: ``forward`` and ``backward`` on torch tensors."""

    def __init__(self, scale: float, causal: bool):
        self.scale = float(scale)
        self.causal = bool(causal)

    def forward(self, q, k, v, residual: bool = True):
        """Returns (o, lse, o_lo); o_lo is None when ``residual`` is False."""
        B, H, N, d = q.shape
        o = torch.empty_like(q)
        o_lo = torch.empty_like(q) if residual else None
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
        fa_fwd(q, k, v, o, lse, self.scale, self.causal, o_lo=o_lo)
        return o, lse, o_lo

    def backward(self, q, k, v, o, lse, dO, o_lo=None):
        B, H, N, d = q.shape
        ws = torch.empty(fa_bwd_workspace_bytes(B, H, N, d), dtype=torch.uint8, device=q.device)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        fa_bwd(q, k, v, o, dO, lse, dq, dk, dv, self.scale, self.causal, ws, o_lo=o_lo)
        return dq, dk, dv


def fa_fwd_dropout(q, k, v, o, lse, scale: float, causal: bool, rate: float, seed: int, offset: int = 0,
                   stream=None, o_lo=None) -> None:
    """Forward with dropout on the attention probabilities (``fa_fwd_dropout``)."""
    B, H, N, d = q.shape
    for nm, t in (("q", q), ("k", k), ("v", v), ("o", o)):
        _check(t, nm, torch.bfloat16, (B, H, N, d))
    _check(lse, "lse", torch.float32, (B, H, N))
    if o_lo is not None:
        _check(o_lo, "o_lo", torch.bfloat16, (B, H, N, d))
    rc = lib().fa_fwd_dropout(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                              o_lo.data_ptr() if o_lo is not None else None, lse.data_ptr(), B, H, N, d,
                              float(scale), int(bool(causal)), float(rate), int(seed) & (2**64 - 1),
                              int(offset) & 0xFFFFFFFF, _stream_handle(stream))
    if rc != FA_OK:
        raise FaError(rc, "fa_fwd_dropout")


def fa_bwd_dropout(q, k, v, o, dO, lse, dq, dk, dv, scale: float, causal: bool, rate: float, seed: int,
                   workspace, offset: int = 0, stream=None, o_lo=None) -> None:
    """Backward of ``fa_fwd_dropout`` (the mask is regenerated from rate, seed and offset)."""
    B, H, N, d = q.shape
    for nm, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dO", dO), ("dq", dq), ("dk", dk), ("dv", dv)):
        _check(t, nm, torch.bfloat16, (B, H, N, d))
    _check(lse, "lse", torch.float32, (B, H, N))
    _check(workspace, "workspace", torch.uint8)
    if o_lo is not None:
        _check(o_lo, "o_lo", torch.bfloat16, (B, H, N, d))
    rc = lib().fa_bwd_dropout(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                              o_lo.data_ptr() if o_lo is not None else None, dO.data_ptr(), lse.data_ptr(),
                              dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, N, d, float(scale),
                              int(bool(causal)), float(rate), int(seed) & (2**64 - 1), int(offset) & 0xFFFFFFFF,
                              workspace.data_ptr(), workspace.numel(), _stream_handle(stream))
    if rc != FA_OK:
        raise FaError(rc, "fa_bwd_dropout")


def fa_dropout_mask(B: int, H: int, N: int, rate: float, seed: int, offset: int, mask, stream=None) -> None:
    """keep[b, h, i, j] in {0, 1} into the uint8 CUDA tensor ``mask`` [B,H,N,N]."""
    _check(mask, "mask", torch.uint8, (B, H, N, N))
    rc = lib().fa_dropout_mask(B, H, N, float(rate), int(seed) & (2**64 - 1), int(offset) & 0xFFFFFFFF,
                               mask.data_ptr(), _stream_handle(stream))
    if rc != FA_OK:
        raise FaError(rc, "fa_dropout_mask")
