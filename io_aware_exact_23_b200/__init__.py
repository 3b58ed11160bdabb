"""B200-native exact attention (FlashAttention-style), forward and backward.

The hot path lives in ``csrc/`` as hand-written sm_100a CUDA kernels behind the
C-ABI library ``libfa.so`` (declared in ``include/fa.h``).  ``binding`` is a thin
ctypes layer over that library: it marshals torch tensors into raw pointers and
does no arithmetic.  Importing ``binding`` (or calling ``fa_fwd``/``fa_bwd``
from here) raises if the library was not built -- there is no CPU fallback.
"""
from __future__ import annotations

__all__ = ["fa_fwd", "fa_bwd", "fa_bwd_workspace_bytes", "fa_device_status", "FaError"]


def __getattr__(name):
    if name in __all__:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
