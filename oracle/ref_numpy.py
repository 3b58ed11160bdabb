"""Whole-matrix NumPy fp64 restatement of vanilla attention, for tiny shapes.

TEST INFRASTRUCTURE ONLY.  It exists to cross-check the per-row C loops of
``ref_attn.c`` with differently structured code: here S_0 = scale * Q K^T and
S_1 = softmax(S_0) are materialised as whole N x N matrices, exactly the
three-pass "Vanilla Attention" listing of the FlashAttention review
(mrodiduger), with the 1/sqrt(d) scale and the causal mask added.  The
backward is the matrix form of the chain rule through softmax.
"""
from __future__ import annotations

import numpy as np


def _scores(q, k, scale, causal):
    s = scale * np.einsum("bhid,bhjd->bhij", q, k)
    if causal:
        n = q.shape[2]
        s = np.where(np.tril(np.ones((n, n), dtype=bool)), s, -np.inf)
    return s


def np_fwd(q, k, v, scale, causal):
    """O [B,H,N,d], LSE [B,H,N] and P [B,H,N,N] (fp64)."""
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    s = _scores(q, k, scale, causal)
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=-1, keepdims=True)
    p = e / l
    o = p @ v
    lse = (m + np.log(l))[..., 0]
    return o, lse, p


def np_bwd(q, k, v, dO, scale, causal):
    """dQ, dK, dV [B,H,N,d] (fp64)."""
    q, k, v, dO = (np.asarray(x, dtype=np.float64) for x in (q, k, v, dO))
    _, _, p = np_fwd(q, k, v, scale, causal)
    dv = np.swapaxes(p, -1, -2) @ dO
    dp = dO @ np.swapaxes(v, -1, -2)
    ds = p * (dp - (p * dp).sum(axis=-1, keepdims=True))
    dq = scale * ds @ k
    dk = scale * np.swapaxes(ds, -1, -2) @ q
    return dq, dk, dv
