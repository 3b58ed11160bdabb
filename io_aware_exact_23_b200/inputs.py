"""Seeded synthetic inputs and the named workloads.

This module is shared by the tests, the bench and the smoke check, and it
holds none of attention's arithmetic: it only draws random tensors and names
shapes.  Recipe (the pages name no dataset): every tensor is [B, H, N, d],
drawn iid N(0, 1) in fp32 from one CPU ``torch.Generator`` seeded with
``seed``, in the order Q, K, V, dO, then rounded to bf16 (round to nearest
even).  The stress variant multiplies Q and K by 8 after rounding; a power of
two is exact in bf16, so the logits grow 64x and exercise the online-softmax
rescale.  scale = 1/sqrt(d).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool
    qk_mult: float = 1.0
    seed: int = 0
    tags: tuple = field(default_factory=tuple)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def fwd_flops(self) -> float:
        """Counted forward FLOPs: 4*B*H*N^2*d, halved when causal."""
        f = 4.0 * self.B * self.H * self.N * self.N * self.d
        return f / 2 if self.causal else f

    def bwd_flops(self) -> float:
        """Counted backward FLOPs: 2.5x the forward count."""
        return 2.5 * self.fwd_flops()

    def elems(self) -> int:
        return self.B * self.H * self.N * self.d


TINY = Workload("tiny_b1h2n256d64", 1, 2, 256, 64, False)
C2 = Workload("b4h16n2048d64", 4, 16, 2048, 64, False)
C3 = Workload("b2h32n4096d128_causal", 2, 32, 4096, 128, True)
C4 = Workload("long_b1h16n32768d128_causal", 1, 16, 32768, 128, True)


def sweep() -> list[Workload]:
    """Constant B*N = 16384 tokens, H = 16, every (d, N, causal, stress) point."""
    out = []
    for d in (64, 128):
        for n in (512, 1024, 2048, 4096, 8192, 16384):
            for causal in (False, True):
                for mult in (1.0, 8.0):
                    tag = ("_causal" if causal else "") + ("_x8" if mult != 1.0 else "")
                    out.append(Workload(f"sweep_b{16384 // n}h16n{n}d{d}{tag}",
                                        16384 // n, 16, n, d, causal, mult))
    return out


CONFIGS = {w.name: w for w in (TINY, C2, C3, C4, *sweep())}


def make_inputs(w: Workload, device="cpu", with_grad_out: bool = True):
    """Q, K, V (and dO) as bf16 [B, H, N, d] tensors, drawn on the CPU then moved."""
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed)
    shape = (w.B, w.H, w.N, w.d)
    names = ("q", "k", "v", "do") if with_grad_out else ("q", "k", "v")
    out = {}
    for nm in names:
        out[nm] = torch.randn(shape, generator=g, dtype=torch.float32).to(torch.bfloat16)
    if w.qk_mult != 1.0:
        out["q"] = out["q"] * w.qk_mult
        out["k"] = out["k"] * w.qk_mult
    if device != "cpu":
        out = {nm: t.to(device) for nm, t in out.items()}
    return out


def make_fp8_inputs(w: Workload, device="cpu"):
    """e4m3 codes of Q, K, V with one fp32 descale factor per head.

    The fp32 draws are those of ``make_inputs`` (same generator, same order,
    before the bf16 rounding; the stress multiplier applies to Q and K).  Per
    (b, h) and tensor, descale = max|x| / 448 (448 is e4m3's largest finite
    value), and the codes are x / descale rounded to nearest even in e4m3
    (torch's float8_e4m3fn conversion), returned as uint8.  The values the
    codes stand for are code_value * descale.
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed)
    shape = (w.B, w.H, w.N, w.d)
    out = {}
    for nm in ("q", "k", "v"):
        x = torch.randn(shape, generator=g, dtype=torch.float32)
        if nm in ("q", "k") and w.qk_mult != 1.0:
            x = x * w.qk_mult
        amax = x.abs().amax(dim=(2, 3)).clamp_min(1e-30)
        descale = amax / 448.0
        codes = (x / descale[:, :, None, None]).to(torch.float8_e4m3fn).view(torch.uint8)
        out[nm] = codes.to(device)
        out["d" + nm] = descale.to(device)
    return out


def make_shape_inputs(B, H, N, d, seed=0, qk_mult=1.0, device="cpu"):
    """Same recipe for an ad-hoc shape (edge-case tests)."""
    return make_inputs(Workload("adhoc", B, H, N, d, False, qk_mult, seed), device=device)


def score_matrix_bytes(B: int, H: int, N: int, elem_bytes: int = 2) -> int:
    """HBM bytes a materialised N x N score matrix would take for B*H heads."""
    return B * H * N * N * elem_bytes
