"""FP8 (e4m3) attention forward: the fp64 reference and the error bound of
rounding P to e4m3 (test infrastructure only, as the rest of ``oracle``).

Reading (the FlashAttention topic page, "FlashAttention-3 (2024)", names FP8
without a scheme): Q, K and V arrive as e4m3 codes with one fp32 descale
factor per head, so the inputs are the exact reals code_value * descale.  The
reference output is exact attention of those dequantised inputs (``ref_fwd``
of ``oracle``).  A kernel that feeds the PV product with P rounded to e4m3
differs from it by that rounding, which ``p_rounding_bound`` bounds element by
element.

e4m3 (the "fn" variant: no infinities): 1 sign bit, 4 exponent bits with bias
7, 3 mantissa bits.  Exponent field e > 0: (1 + m/8) * 2^(e-7); e = 0:
subnormal (m/8) * 2^-6; exponent and mantissa all ones (S.1111.111): NaN.
Largest finite value 448, smallest normal 2^-6, subnormal step 2^-9.

Rounding to nearest even gives, for a value x with |x| >= 2^-6 (normal range),
|round(x) - x| <= 2^-4 |x| (half a unit in the last of 3 mantissa bits), and
below 2^-6 an absolute error of at most 2^-10 (half the subnormal step).
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
E4M3_MIN_NORMAL = 2.0 ** -6
REL_ERR = 2.0 ** -4    # normal range, round to nearest
ABS_ERR = 2.0 ** -10   # subnormal range, round to nearest


def e4m3_values() -> np.ndarray:
    """The 256 e4m3 codes decoded from the bit layout above (NaN at 0x7F, 0xFF)."""
    out = np.empty(256, dtype=np.float64)
    for code in range(256):
        sign = -1.0 if code & 0x80 else 1.0
        e = (code >> 3) & 0xF
        m = code & 0x7
        if e == 0xF and m == 0x7:
            out[code] = np.nan
        elif e == 0:
            out[code] = sign * (m / 8.0) * 2.0 ** -6
        else:
            out[code] = sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return out


_TABLE = e4m3_values()


def dequantize(codes, descale) -> np.ndarray:
    """codes [B, H, N, d] uint8 and descale [B, H] -> fp64 values code * descale."""
    c = np.asarray(codes.cpu().numpy() if hasattr(codes, "cpu") else codes, dtype=np.uint8)
    s = np.asarray(descale.cpu().numpy() if hasattr(descale, "cpu") else descale, dtype=np.float64)
    assert c.ndim == 4 and s.shape == c.shape[:2]
    return _TABLE[c] * s[:, :, None, None]


def ref_fwd_fp8(q8, k8, v8, dq, dk, dv, scale: float, causal: bool, nthreads: int = 0):
    """O and LSE (fp64) of exact attention of the dequantised inputs."""
    from . import ref_fwd
    return ref_fwd(dequantize(q8, dq), dequantize(k8, dk), dequantize(v8, dv), scale, causal, nthreads=nthreads)


def p_rounding_bound(q, k, v, scale: float, causal: bool) -> np.ndarray:
    """Element-wise bound on |O - O_ref| when P is rounded to e4m3 before PV.

    With p_ij = exp(S_ij - max_j S_ij) and l_i = sum_j p_ij (fp64, exact inputs),
    a kernel computes O_i = sum_j round(P_ij) V_j / L_i with P_ij = p_ij * 2^t and
    L_i = l_i * 2^t for some t >= 0 (its running max is at most the true one).
    The rounding error of each P_ij is at most max(2^-4 P_ij, 2^-10), and in the
    units of p that is at most max(2^-4 p_ij, 2^-10 * 2^-t) <= max(2^-4 p_ij, 2^-10).
    Hence |O_ic - O_ref_ic| <= sum_j max(2^-4 p_ij, 2^-10) |V_jc| / l_i.
    Inputs: fp64 [B, H, N, d] (dequantised); returns the bound, same shape.
    """
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    B, H, N, d = q.shape
    out = np.empty_like(q)
    for b in range(B):
        for h in range(H):
            s = scale * (q[b, h] @ k[b, h].T)
            if causal:
                s = np.where(np.tril(np.ones((N, N), dtype=bool)), s, -np.inf)
            p = np.exp(s - s.max(axis=1, keepdims=True))
            l = p.sum(axis=1, keepdims=True)
            err = np.where(p > 0, np.maximum(REL_ERR * p, ABS_ERR), 0.0)
            out[b, h] = (err @ np.abs(v[b, h])) / l
    return out
