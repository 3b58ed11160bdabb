"""CPU fp64 oracle for exact scaled-dot-product attention (forward and backward).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this package; the product path
(``io_aware_exact_23_b200``) never does, and the two share no code.

``ref_attn.c`` holds the arithmetic (plain per-row loops in fp64, see its
header for the passages of the FlashAttention pages it follows); ``fp8.py``
the e4m3 decoder, the FP8 forward's reference and its P-rounding bound;
``ref_numpy.py`` is an independent whole-matrix NumPy restatement used only
to cross-check the C code on tiny shapes.  This module compiles the C file
with gcc on first use and marshals arrays through ctypes.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(closed forms, invariants, finite differences, autograd, hand-derived golden
fixtures), the dropout functions by ``tests/test_dropout_oracle_pins.py`` and
``fp8.py`` by ``tests/test_fp8_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ref_attn.c")
_SRCS = [_SRC, os.path.join(_HERE, "ref_dropout.c")]
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``ref_attn.c`` and ``ref_dropout.c`` into ``liboracle.so`` (plain -O2, IEEE fp64)."""
    if force or not os.path.exists(_LIB) or any(os.path.getmtime(_LIB) < os.path.getmtime(s) for s in _SRCS):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
             "-fno-fast-math", "-ffp-contract=off", *_SRCS, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        D = ctypes.POINTER(ctypes.c_double)
        L = ctypes.POINTER(ctypes.c_long)
        cl, cd, ci = ctypes.c_long, ctypes.c_double, ctypes.c_int
        lib.ref_attn_fwd.argtypes = [D, D, D, D, D, cl, cl, cl, cl, cd, ci, ci]
        lib.ref_attn_bwd.argtypes = [D, D, D, D, D, D, D, cl, cl, cl, cl, cd, ci, ci]
        lib.ref_attn_fwd_rows.argtypes = [D, D, D, cl, cl, cl, cl, cd, ci, L, L, cl, D, D, ci]
        lib.ref_attn_dq_rows.argtypes = [D, D, D, D, cl, cl, cl, cl, cd, ci, L, L, cl, D, ci]
        lib.ref_attn_dkdv_rows.argtypes = [D, D, D, D, cl, cl, cl, cl, cd, ci, cl, L, cl, D, D, ci]
        for f in (lib.ref_attn_fwd, lib.ref_attn_bwd, lib.ref_attn_fwd_rows, lib.ref_attn_dq_rows,
                  lib.ref_attn_dkdv_rows):
            f.restype = ctypes.c_int
        U32 = ctypes.POINTER(ctypes.c_uint32)
        u64, u32 = ctypes.c_uint64, ctypes.c_uint32
        lib.ref_philox4x32_10.argtypes = [U32, U32, U32]
        lib.ref_philox4x32_10.restype = None
        lib.ref_dropout_mask.argtypes = [cl, cl, u64, u32, u32, ctypes.POINTER(ctypes.c_uint8)]
        lib.ref_dropout_mask.restype = None
        lib.ref_attn_fwd_dropout.argtypes = [D, D, D, D, D, cl, cl, cl, cd, ci, u64, u32, u32, cl]
        lib.ref_attn_fwd_dropout.restype = ci
        lib.ref_attn_bwd_dropout.argtypes = [D, D, D, D, D, D, D, cl, cl, cl, cd, ci, u64, u32, u32, cl]
        lib.ref_attn_bwd_dropout.restype = ci
        _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    """Exact widening of float inputs (bf16/fp32/fp64 tensors or arrays) to fp64."""
    if hasattr(x, "detach"):  # torch tensor: widen in torch (exact for bf16), then view
        import torch
        x = x.detach().to("cpu", torch.float64).contiguous().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _shape4(q):
    if q.ndim != 4:
        raise ValueError("expected a [B, H, N, d] tensor")
    return q.shape


def ref_fwd(q, k, v, scale: float, causal: bool, nthreads: int = 0):
    """O [B,H,N,d] and LSE [B,H,N] in fp64 (vanilla attention, safe softmax)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = _shape4(q)
    assert k.shape == q.shape and v.shape == q.shape
    o = np.empty_like(q)
    lse = np.empty((B, H, N), dtype=np.float64)
    rc = _load().ref_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                              B, H, N, d, float(scale), int(bool(causal)), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"ref_attn_fwd failed ({rc})")
    return o, lse


def ref_bwd(q, k, v, dO, scale: float, causal: bool, nthreads: int = 0):
    """dQ, dK, dV [B,H,N,d] in fp64 for the upstream gradient dO."""
    q, k, v, dO = _f64(q), _f64(k), _f64(v), _f64(dO)
    B, H, N, d = _shape4(q)
    assert k.shape == q.shape and v.shape == q.shape and dO.shape == q.shape
    dq, dk, dv = np.empty_like(q), np.empty_like(q), np.empty_like(q)
    rc = _load().ref_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(dO), _ptr(dq), _ptr(dk), _ptr(dv),
                              B, H, N, d, float(scale), int(bool(causal)), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"ref_attn_bwd failed ({rc})")
    return dq, dk, dv


def _samples(samp_bh, samp_row):
    sb = np.ascontiguousarray(np.asarray(samp_bh, dtype=np.int64)).astype(np.dtype("l"))
    sr = np.ascontiguousarray(np.asarray(samp_row, dtype=np.int64)).astype(np.dtype("l"))
    assert sb.shape == sr.shape and sb.ndim == 1
    return sb, sr


def ref_fwd_rows(q, k, v, scale: float, causal: bool, samp_bh, samp_row, nthreads: int = 0):
    """O rows [n, d] and LSE [n] at the sampled (flat head index, query row) pairs."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = _shape4(q)
    sb, sr = _samples(samp_bh, samp_row)
    n = sb.shape[0]
    o = np.empty((n, d), dtype=np.float64)
    lse = np.empty((n,), dtype=np.float64)
    Lp = ctypes.POINTER(ctypes.c_long)
    rc = _load().ref_attn_fwd_rows(_ptr(q), _ptr(k), _ptr(v), B, H, N, d, float(scale),
                                   int(bool(causal)), sb.ctypes.data_as(Lp), sr.ctypes.data_as(Lp),
                                   n, _ptr(o), _ptr(lse), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"ref_attn_fwd_rows failed ({rc})")
    return o, lse


def ref_dq_rows(q, k, v, dO, scale: float, causal: bool, samp_bh, samp_row, nthreads: int = 0):
    """dQ rows [n, d] at the sampled (flat head index, query row) pairs."""
    q, k, v, dO = _f64(q), _f64(k), _f64(v), _f64(dO)
    B, H, N, d = _shape4(q)
    sb, sr = _samples(samp_bh, samp_row)
    n = sb.shape[0]
    dq = np.empty((n, d), dtype=np.float64)
    Lp = ctypes.POINTER(ctypes.c_long)
    rc = _load().ref_attn_dq_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(dO), B, H, N, d, float(scale),
                                  int(bool(causal)), sb.ctypes.data_as(Lp), sr.ctypes.data_as(Lp),
                                  n, _ptr(dq), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"ref_attn_dq_rows failed ({rc})")
    return dq


def ref_dkdv_rows(q, k, v, dO, scale: float, causal: bool, head: int, key_rows, nthreads: int = 0):
    """dK, dV rows [n, d] of one head (flat index) at the given key rows."""
    q, k, v, dO = _f64(q), _f64(k), _f64(v), _f64(dO)
    B, H, N, d = _shape4(q)
    kr = np.ascontiguousarray(np.asarray(key_rows, dtype=np.int64)).astype(np.dtype("l"))
    n = kr.shape[0]
    dk = np.empty((n, d), dtype=np.float64)
    dv = np.empty((n, d), dtype=np.float64)
    Lp = ctypes.POINTER(ctypes.c_long)
    rc = _load().ref_attn_dkdv_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(dO), B, H, N, d, float(scale),
                                    int(bool(causal)), int(head), kr.ctypes.data_as(Lp), n,
                                    _ptr(dk), _ptr(dv), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"ref_attn_dkdv_rows failed ({rc})")
    return dk, dv


# ------------------------------------------------------------------ dropout

def dropout_threshold(rate: float) -> int:
    """T = floor(rate * 256), with the rate as the 32-bit float the C interface takes:
    a key is dropped when its 8-bit draw is below T."""
    r = float(np.float32(rate))
    if not (0.0 <= r < 1.0):
        raise ValueError("dropout rate must be in [0, 1)")
    return int(np.floor(r * 256.0))


def philox4x32_10(counter, key):
    """Philox4x32-10 of a 4-word counter and a 2-word key (``ref_dropout.c``)."""
    c = (ctypes.c_uint32 * 4)(*[int(x) & 0xFFFFFFFF for x in counter])
    k = (ctypes.c_uint32 * 2)(*[int(x) & 0xFFFFFFFF for x in key])
    out = (ctypes.c_uint32 * 4)()
    _load().ref_philox4x32_10(c, k, out)
    return [int(x) for x in out]


def dropout_mask(BH: int, N: int, seed: int, offset: int, rate: float) -> np.ndarray:
    """keep[bh, i, j] (uint8 0/1) of the dropout mask, [BH, N, N]."""
    keep = np.zeros((BH, N, N), dtype=np.uint8)
    _load().ref_dropout_mask(BH, N, seed, offset, dropout_threshold(rate),
                             keep.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)))
    return keep


def ref_fwd_dropout(q, k, v, scale: float, causal: bool, rate: float, seed: int, offset: int, head0: int = 0):
    """O [B,H,N,d] and LSE [B,H,N] in fp64 with dropout on the attention probabilities.

    ``head0``: global index b*H + h of the first head passed (when checking some
    heads of a larger workload on their own)."""
    B, H, N, d = _shape4(q)
    qq, kk, vv = _f64(q), _f64(k), _f64(v)
    o = np.zeros((B, H, N, d)); lse = np.zeros((B, H, N))
    rc = _load().ref_attn_fwd_dropout(_ptr(qq), _ptr(kk), _ptr(vv), _ptr(o), _ptr(lse), B * H, N, d, float(scale),
                                      int(bool(causal)), seed, offset, dropout_threshold(rate), head0)
    if rc != 0:
        raise MemoryError("ref_attn_fwd_dropout")
    return o, lse


def ref_bwd_dropout(q, k, v, do, scale: float, causal: bool, rate: float, seed: int, offset: int,
                    head0: int = 0):
    """dQ, dK, dV [B,H,N,d] in fp64 with dropout on the attention probabilities (``head0``
    as for ``ref_fwd_dropout``)."""
    B, H, N, d = _shape4(q)
    qq, kk, vv, gg = _f64(q), _f64(k), _f64(v), _f64(do)
    dq, dk, dv = (np.zeros((B, H, N, d)) for _ in range(3))
    rc = _load().ref_attn_bwd_dropout(_ptr(qq), _ptr(kk), _ptr(vv), _ptr(gg), _ptr(dq), _ptr(dk), _ptr(dv),
                                      B * H, N, d, float(scale), int(bool(causal)), seed, offset,
                                      dropout_threshold(rate), head0)
    if rc != 0:
        raise MemoryError("ref_attn_bwd_dropout")
    return dq, dk, dv
