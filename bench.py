#!/usr/bin/env python
"""Throughput of one fused attention training step (forward + backward) on B200.

A step is one pass of the whole hot path over one batch: ``fa_fwd`` (O, LSE and
O's rounding residual) then ``fa_bwd`` (D preprocess, dK/dV/dQ kernel, dQ
conversion) on the
workload B=2, H=32, N=4096, d=128, causal -- the first configuration at the
N >= 4096, d = 128 point where the throughput targets are stated.  Inputs are
synthetic (seeded N(0,1) rounded to bf16) and already resident in HBM when the
timed region starts; Q, K, V and dO alone are 268 MB, larger than the 126 MB L2,
so no L2 flush is inserted between steps.

Counted FLOPs: forward 4*B*H*N^2*d, backward 2.5x that, both halved for causal.

Launch: ``python bench.py --gpus N --steps K --warmup W`` (one rank per GPU
under torchrun for N > 1; every rank runs the same workload: weak scaling, no
data-path collective).  Prints one JSON line on rank 0.
``--impl reference`` times the CPU fp64 oracle instead (rank 0 only);
``--impl vanilla`` times standard attention (S and P in HBM) on one GPU;
``--dropout RATE`` times the step with fused dropout on the probabilities;
``--deterministic`` times the step with the deterministic backward;
``--sweep`` prints one line per workload (forward and backward separately);
``--fp8`` times the e4m3 forward (fa_fwd_fp8) on the workload;
``--max-n`` finds the longest sequence each library runs (fwd + bwd, B=1, H=16,
d=128, causal): this library and standard attention (``libfa_vanilla.so``).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attention fwd and fwd+bwd TFLOP/s (bf16, 1×B200) and % of tensor peak"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# Device code of each timed kernel (a changed file invalidates its stored ncu traffic).
KERNEL_SOURCES = {
    "fa_fwd_kernel": ["io_aware_exact_23_b200/csrc/ptx.cuh", "io_aware_exact_23_b200/csrc/fa_fwd.cuh"],
    "fa_bwd_kernel": ["io_aware_exact_23_b200/csrc/ptx.cuh", "io_aware_exact_23_b200/csrc/fa_bwd.cuh"],
}


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference", "vanilla"], default="ours")
    ap.add_argument("--workload", default="b2h32n4096d128_causal")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-budget-s", type=float, default=12.0,
                    help="seconds of oracle work for the cpu_baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sweep", action="store_true",
                    help="one JSON line per workload (tiny, C2, C3, long and the non-stress sweep points): "
                         "forward and backward TFLOP/s, fraction of peak, peak HBM vs the N^2 score size; 1 GPU")
    ap.add_argument("--deterministic", action="store_true",
                    help="time the step with fa_bwd_deterministic (dQ in a fixed summation order)")
    ap.add_argument("--dropout", type=float, default=0.0,
                    help="time the fused-dropout step (fa_fwd_dropout + fa_bwd_dropout) at this rate, 1 GPU")
    ap.add_argument("--fp8", action="store_true",
                    help="time the e4m3 forward (fa_fwd_fp8) on the workload (d = 128), 1 GPU")
    ap.add_argument("--max-n", action="store_true",
                    help="longest sequence (B=1, H=16, d=128, causal, fwd + bwd) that runs, for this library and "
                         "for standard attention; 1 GPU")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def source_sha(kernel: str) -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES.get(kernel, []):
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def stored_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu capture, if the kernels have not changed since."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    for r in rec.get("records", []):
        if r.get("kernel") == kernel and r.get("workload") == workload and r.get("source_sha") == source_sha(kernel):
            return r.get("dram_bytes_per_launch")
    return None


class ClockSampler:
    """nvidia-smi clocks/throttle sampling; keeps samples taken inside [t0, t1]."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str | None):
        self.samples = []
        self.proc = None
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "50"]
        if gpu_id:
            cmd[1:1] = ["-i", gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), line.strip()))

    def wait_ready(self, timeout: float = 10.0):
        """Block until nvidia-smi has produced its first sample (or timeout)."""
        t_end = time.time() + timeout
        while self.proc is not None and not self.samples and time.time() < t_end:
            time.sleep(0.02)

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0: float, t1: float):
        # Samples inside the timed region; if it was shorter than the sampling
        # period, the samples within a quarter second of it.
        window = "timed region"
        if not any(t0 <= ts <= t1 for ts, _ in self.samples):
            t0, t1, window = t0 - 0.25, t1 + 0.25, "timed region +-0.25 s"
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ts, line in self.samples:
            if not (t0 <= ts <= t1):
                continue
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm), "window": window}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def rank_workload(w, rank: int):
    """Rank r's shard of the global batch: the same shape, its own seed (r)."""
    import dataclasses
    return dataclasses.replace(w, seed=w.seed + rank)


def reduce_max(values, dist, device):
    """Element-wise max over ranks (device timing: the slowest rank sets the time)."""
    import torch
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return list(values)
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def cpu_baseline_sample(w, budget_s: float):
    """Time the oracle (as it stands) on whole heads of the workload until the budget is spent."""
    import numpy as np
    import torch

    import oracle
    from io_aware_exact_23_b200.inputs import make_inputs
    t = make_inputs(w)  # CPU tensors
    cores = os.cpu_count() or 1
    oracle.build()
    heads, flops, secs = 0, 0.0, 0.0
    per_head = (w.fwd_flops() + w.bwd_flops()) / (w.B * w.H)
    for bh in range(w.B * w.H):
        b, h = divmod(bh, w.H)
        sl = {k: v[b:b + 1, h:h + 1] for k, v in t.items()}
        t0 = time.perf_counter()
        oracle.ref_fwd(sl["q"], sl["k"], sl["v"], w.scale, w.causal, nthreads=cores)
        oracle.ref_bwd(sl["q"], sl["k"], sl["v"], sl["do"], w.scale, w.causal, nthreads=cores)
        secs += time.perf_counter() - t0
        heads += 1
        flops += per_head
        if secs >= budget_s:
            break
    del np, torch
    return {"value": flops / secs / 1e12, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{heads} of {w.B * w.H} heads (b,h in order) of {w.name}, forward + backward, "
                      f"fp64 C oracle with {cores} threads, {secs:.1f} s"}


def run_reference(args, w, world, rank):
    """--impl reference: the CPU oracle on the same workload, one head per step (rank 0 only)."""
    if rank != 0:
        return 0
    import oracle
    from io_aware_exact_23_b200.inputs import make_inputs
    cores = os.cpu_count() or 1
    oracle.build()
    t = make_inputs(w)
    per_head = (w.fwd_flops() + w.bwd_flops()) / (w.B * w.H)
    BH = w.B * w.H

    def step(s):
        b, h = divmod(s % BH, w.H)
        sl = {k: v[b:b + 1, h:h + 1] for k, v in t.items()}
        oracle.ref_fwd(sl["q"], sl["k"], sl["v"], w.scale, w.causal, nthreads=cores)
        oracle.ref_bwd(sl["q"], sl["k"], sl["v"], sl["do"], w.scale, w.causal, nthreads=cores)

    for s in range(args.warmup):
        step(s)
    t0 = time.perf_counter()
    done = 0
    for s in range(args.steps):
        step(args.warmup + s)
        done += 1
        if time.perf_counter() - t0 > 240.0:  # keep the arm within a few minutes
            break
    secs = time.perf_counter() - t0
    value = per_head * done / secs / 1e12
    sample = (f"one (b,h) head of {w.name} per step (fwd + bwd, fp64 C oracle, {cores} threads), "
              f"{done} steps")
    line = {"metric": METRIC, "value": value, "unit": UNIT, "impl": "reference", "n_gpus": world,
            "steps": done, "warmup": args.warmup, "ms_per_step": secs / done * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal,
                       "step": "one head of the workload (CPU oracle)"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def l2_note(w) -> str:
    """How the timed steps stay honest about L2 (126 MB): inputs larger than L2, else flushed."""
    mb = 4 * w.B * w.H * w.N * w.d * 2 / 1e6  # Q, K, V, dO in bf16
    if mb > 126:
        return f"no flush: Q, K, V, dO total {mb:.0f} MB, larger than the 126 MB L2"
    return f"inputs total {mb:.0f} MB (< 126 MB L2): each step's outputs and workspace pass through L2"


def run_vanilla(args, w):
    """--impl vanilla (1 GPU): standard attention with S and P materialised in HBM
    (libfa_vanilla.so: cuBLAS GEMMs + this library's row softmax kernels), timed
    on the same workload and FLOP convention as the IO-aware path."""
    import torch
    from io_aware_exact_23_b200 import vanilla
    from io_aware_exact_23_b200.inputs import make_inputs
    dev = torch.device("cuda:0")
    t = make_inputs(w, device=dev)
    q, k, v, dO = t["q"], t["k"], t["v"], t["do"]
    B, H, N, d = q.shape
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    ws = torch.empty(vanilla.workspace_bytes(B, H, N, d), dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()
    torch.cuda.reset_peak_memory_stats(dev)
    mk = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731

    def step(ev=None):
        if ev is not None:
            ev[0].record()
        vanilla.fwd(q, k, v, o, lse, w.scale, w.causal, ws)
        if ev is not None:
            ev[1].record()
        vanilla.bwd(q, k, v, o, dO, lse, dq, dk, dv, w.scale, w.causal, ws)
        if ev is not None:
            ev[2].record()

    for _ in range(max(args.warmup, 0)):
        step()
    K = args.steps
    evs = [(mk(), mk(), mk()) for _ in range(K)]
    start, end = mk(), mk()
    torch.cuda.synchronize()
    start.record()
    for s_ in range(K):
        step(evs[s_])
    end.record()
    torch.cuda.synchronize()
    ms = start.elapsed_time(end)
    fwd_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    bwd_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    flops = w.fwd_flops() + w.bwd_flops()
    line = {"metric": METRIC, "value": flops * K / (ms / 1e3) / 1e12, "unit": UNIT, "impl": "vanilla", "n_gpus": 1,
            "steps": K, "warmup": args.warmup, "ms_per_step": ms / K, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal,
                       "step": "standard attention fwd + bwd, S (fp32) and P (bf16) materialised in HBM"},
            "fwd_tflops": w.fwd_flops() / (fwd_ms / 1e3) / 1e12, "bwd_tflops": w.bwd_flops() / (bwd_ms / 1e3) / 1e12,
            "fwd_ms": fwd_ms, "bwd_ms": bwd_ms, "workspace_bytes": ws.numel(),
            "peak_hbm_bytes": torch.cuda.max_memory_allocated(dev), "gpu_launches": 2 * K,
            "library_gemms_per_step": 6}
    print(json.dumps(line), flush=True)
    return 0


def run_variant(args, w):
    """--dropout RATE or --deterministic (1 GPU): the IO-aware step with fused
    dropout on the probabilities, or with the deterministic backward (dQ summed
    over key tiles in a fixed order by its own kernel)."""
    import torch
    from io_aware_exact_23_b200 import binding as fa
    from io_aware_exact_23_b200.inputs import make_inputs
    dev = torch.device("cuda:0")
    t = make_inputs(w, device=dev)
    q, k, v, dO = t["q"], t["k"], t["v"], t["do"]
    B, H, N, d = q.shape
    o, o_lo = torch.empty_like(q), torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    ws = torch.empty(fa.fa_bwd_workspace_bytes(B, H, N, d), dtype=torch.uint8, device=dev)
    mk = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    seed = 0x5EED

    def step(s_, ev=None, plain_bwd=False):
        if ev is not None:
            ev[0].record()
        if args.deterministic:
            fa.fa_fwd(q, k, v, o, lse, w.scale, w.causal, o_lo=o_lo)
        else:
            fa.fa_fwd_dropout(q, k, v, o, lse, w.scale, w.causal, args.dropout, seed, s_, o_lo=o_lo)
        if ev is not None:
            ev[1].record()
        if plain_bwd:
            fa.fa_bwd(q, k, v, o, dO, lse, dq, dk, dv, w.scale, w.causal, ws, o_lo=o_lo)
        elif args.deterministic:
            fa.fa_bwd_deterministic(q, k, v, o, dO, lse, dq, dk, dv, w.scale, w.causal, ws, o_lo=o_lo)
        else:
            fa.fa_bwd_dropout(q, k, v, o, dO, lse, dq, dk, dv, w.scale, w.causal, args.dropout, seed, ws,
                              offset=s_, o_lo=o_lo)
        if ev is not None:
            ev[2].record()

    for s_ in range(max(args.warmup, 0)):
        step(s_)
    K = args.steps
    evs = [(mk(), mk(), mk()) for _ in range(K)]
    start, end = mk(), mk()
    torch.cuda.synchronize()
    start.record()
    for s_ in range(K):
        step(args.warmup + s_, evs[s_])
    end.record()
    torch.cuda.synchronize()
    if fa.fa_device_status() != 0:
        raise SystemExit("bench.py: device status error")
    ms = start.elapsed_time(end)
    fwd_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    bwd_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    extra = {}
    if args.deterministic:
        # context, outside the timed region: the same steps with fa_bwd (dQ added in arrival order)
        pev = [(mk(), mk(), mk()) for _ in range(K)]
        for s_ in range(K):
            step(s_, pev[s_], plain_bwd=True)
        torch.cuda.synchronize()
        extra["bwd_ms_fa_bwd"] = statistics.mean(e[1].elapsed_time(e[2]) for e in pev)
        extra["bwd_ms"] = bwd_ms
    peaks, peak_kind = load_peaks()
    peak = float(peaks["bf16_tflops"])
    flops = w.fwd_flops() + w.bwd_flops()
    fwd_tf, bwd_tf = w.fwd_flops() / (fwd_ms / 1e3) / 1e12, w.bwd_flops() / (bwd_ms / 1e3) / 1e12
    line = {"metric": METRIC, "value": flops * K / (ms / 1e3) / 1e12, "unit": UNIT, "impl": "ours", "n_gpus": 1,
            "steps": K, "warmup": args.warmup, "ms_per_step": ms / K, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal,
                       "dropout": args.dropout, "deterministic": bool(args.deterministic), "l2": l2_note(w),
                       "step": ("fa_fwd + fa_bwd_deterministic" if args.deterministic else
                                "fa_fwd_dropout + fa_bwd_dropout (a new mask per step: offset = step)")},
            "fwd_tflops": fwd_tf, "bwd_tflops": bwd_tf, "fwd_frac_of_peak": fwd_tf / peak,
            "bwd_frac_of_peak": bwd_tf / peak, "peak_kind": peak_kind, "gpu_launches": 4 * K, **extra}
    print(json.dumps(line), flush=True)
    return 0


def run_sweep(args):
    """--sweep: fa_fwd and fa_bwd (the default entry points) timed per workload with CUDA events."""
    import torch
    from io_aware_exact_23_b200 import binding as fa
    from io_aware_exact_23_b200.inputs import C2, C3, C4, TINY, make_inputs, score_matrix_bytes, sweep
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    torch.zeros(1, device=dev)  # create the context before the memory statistics are touched
    peaks, peak_kind = load_peaks()
    peak = float(peaks["bf16_tflops"])
    mk = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    for w in [TINY, C2, C3, C4] + [x for x in sweep() if x.qk_mult == 1.0]:
        torch.cuda.empty_cache()
        torch.cuda.reset_peak_memory_stats(dev)
        t = make_inputs(w, device=dev)
        q, k, v, dO = t["q"], t["k"], t["v"], t["do"]
        B, H, N, d = q.shape
        o, lse = torch.empty_like(q), torch.empty((B, H, N), dtype=torch.float32, device=dev)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
        ws = torch.empty(fa.fa_bwd_workspace_bytes(B, H, N, d), dtype=torch.uint8, device=dev)
        reps = max(3, min(50, int(2e12 / max(w.fwd_flops(), 1.0))))
        for _ in range(3):
            fa.fa_fwd(q, k, v, o, lse, w.scale, w.causal)
            fa.fa_bwd(q, k, v, o, dO, lse, dq, dk, dv, w.scale, w.causal, ws)
        e = [mk() for _ in range(3)]
        e[0].record()
        for _ in range(reps):
            fa.fa_fwd(q, k, v, o, lse, w.scale, w.causal)
        e[1].record()
        for _ in range(reps):
            fa.fa_bwd(q, k, v, o, dO, lse, dq, dk, dv, w.scale, w.causal, ws)
        e[2].record()
        torch.cuda.synchronize()
        if fa.fa_device_status() != 0:
            raise SystemExit(f"bench.py: device status error on {w.name}")
        fwd_ms, bwd_ms = e[0].elapsed_time(e[1]) / reps, e[1].elapsed_time(e[2]) / reps
        fwd_tf, bwd_tf = w.fwd_flops() / (fwd_ms / 1e3) / 1e12, w.bwd_flops() / (bwd_ms / 1e3) / 1e12
        print(json.dumps({"workload": w.name, "B": B, "H": H, "N": N, "d": d, "causal": w.causal, "reps": reps,
                          "fwd_ms": fwd_ms, "bwd_ms": bwd_ms, "fwd_tflops": fwd_tf, "bwd_tflops": bwd_tf,
                          "fwd_frac_of_peak": fwd_tf / peak, "bwd_frac_of_peak": bwd_tf / peak,
                          "peak_kind": peak_kind, "peak_hbm_bytes": torch.cuda.max_memory_allocated(dev),
                          "score_matrix_bytes_bf16": score_matrix_bytes(B, H, N), "l2": l2_note(w)}), flush=True)
        del t, q, k, v, dO, o, lse, dq, dk, dv, ws
    return 0


def run_fp8(args, w):
    """--fp8 (1 GPU): the e4m3 forward, fa_fwd_fp8, timed with CUDA events.  Its
    peak is the measured bf16 dense peak x 2 (the nominal e4m3 : bf16 ratio of
    the tensor cores)."""
    import torch
    from io_aware_exact_23_b200 import binding as fa
    from io_aware_exact_23_b200.inputs import make_fp8_inputs
    if w.d != 128:
        raise SystemExit("bench.py: the e4m3 forward takes d = 128")
    dev = torch.device("cuda:0")
    t = make_fp8_inputs(w, device=dev)
    B, H, N, d = w.B, w.H, w.N, w.d
    o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)

    def step():
        fa.fa_fwd_fp8(t["q"], t["k"], t["v"], t["dq"], t["dk"], t["dv"], o, lse, w.scale, w.causal)

    for _ in range(max(args.warmup, 0)):
        step()
    K = args.steps
    mk = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    start, end = mk(), mk()
    torch.cuda.synchronize()
    start.record()
    for _ in range(K):
        step()
    end.record()
    torch.cuda.synchronize()
    if fa.fa_device_status() != 0:
        raise SystemExit("bench.py: device status error")
    ms = start.elapsed_time(end) / K
    peaks, peak_kind = load_peaks()
    peak = 2.0 * float(peaks["bf16_tflops"])
    tf = w.fwd_flops() / (ms / 1e3) / 1e12
    in_bytes = 3 * B * H * N * d
    line = {"metric": METRIC, "value": tf, "unit": UNIT, "impl": "ours", "n_gpus": 1, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "e4m3 in, fp32 accumulate, bf16 out", "data": "synthetic",
            "config": {"workload": w.name, "B": B, "H": H, "N": N, "d": d, "causal": w.causal,
                       "step": "fa_fwd_fp8 (forward only)", "l2": f"inputs {in_bytes / 1e6:.0f} MB"},
            "roofline": {"bound": "tensor", "kernel": "fa_fwd_kernel<128, causal, 0, fp8>", "achieved": tf,
                         "peak": peak, "unit": "TFLOP/s", "frac": tf / peak,
                         "peak_kind": f"e4m3 dense = 2 x bf16 dense burst ({peak_kind}), the nominal ratio"},
            "gpu_launches": K}
    print(json.dumps(line), flush=True)
    return 0


def run_max_n(args):
    """--max-n (1 GPU): the longest sequence that runs one fwd + bwd step at B=1,
    H=16, d=128, causal -- for this library (fa_fwd with the residual + fa_bwd)
    and for standard attention (libfa_vanilla.so, S and P in HBM).  N doubles
    from 8192 until the step cannot run (the allocation fails, or the library
    refuses the shape); the largest N whose tensors allocate is then bisected
    to a multiple of 1024, and the step is run there.  Inputs are N(0,1) bf16
    drawn on the device from a seeded generator (a capacity probe: only the
    sizes matter)."""
    import torch
    from io_aware_exact_23_b200 import binding as fa
    from io_aware_exact_23_b200 import vanilla
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    torch.zeros(1, device=dev)
    total = torch.cuda.get_device_properties(dev).total_memory
    B, H, d, scale = 1, 16, 128, 1.0 / 128 ** 0.5

    def alloc(impl, N):
        """The step's tensors, or the reason they cannot exist."""
        if impl == "ours":
            wsb = fa.fa_bwd_workspace_bytes(B, H, N, d)
            if wsb == 0:
                return None, "refused by the library: B*H*N*d >= 2^31 elements per tensor"
        else:
            wsb = vanilla.workspace_bytes(B, H, N, d)
            if wsb == 0:
                return None, "refused by the library"
        try:
            g = torch.Generator(device=dev)
            g.manual_seed(N)
            T = {nm: torch.randn((B, H, N, d), generator=g, device=dev, dtype=torch.bfloat16)
                 for nm in ("q", "k", "v", "do")}
            for nm in ("o", "dq", "dk", "dv") + (("o_lo",) if impl == "ours" else ()):
                T[nm] = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev)
            T["lse"] = torch.empty((B, H, N), dtype=torch.float32, device=dev)
            T["ws"] = torch.empty(wsb, dtype=torch.uint8, device=dev)
            return T, None
        except torch.cuda.OutOfMemoryError:
            return None, "out of memory (torch allocation)"

    def run(impl, N, T):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        try:
            e0.record()
            if impl == "ours":
                fa.fa_fwd(T["q"], T["k"], T["v"], T["o"], T["lse"], scale, True, o_lo=T["o_lo"])
                fa.fa_bwd(T["q"], T["k"], T["v"], T["o"], T["do"], T["lse"], T["dq"], T["dk"], T["dv"], scale, True,
                          T["ws"], o_lo=T["o_lo"])
            else:
                vanilla.fwd(T["q"], T["k"], T["v"], T["o"], T["lse"], scale, True, T["ws"])
                vanilla.bwd(T["q"], T["k"], T["v"], T["o"], T["do"], T["lse"], T["dq"], T["dk"], T["dv"], scale, True,
                            T["ws"])
            e1.record()
            torch.cuda.synchronize()
        except Exception as ex:  # a library status code (e.g. cuBLAS could not allocate)
            torch.cuda.synchronize()
            return None, f"call failed: {ex}"
        if impl == "ours" and fa.fa_device_status() != 0:
            return None, "device status error"
        finite = bool(torch.isfinite(T["dq"].float()).all() and torch.isfinite(T["o"].float()).all())
        return {"ms": e0.elapsed_time(e1), "finite": finite}, None

    def free():
        torch.cuda.synchronize()
        torch.cuda.empty_cache()

    for impl in ("ours", "vanilla"):
        tried = []
        N, ok_n, fail_n, fail_why = 8192, None, None, None
        while True:
            T, why = alloc(impl, N)
            r = None
            if T is not None:
                torch.cuda.reset_peak_memory_stats(dev)
                r, why = run(impl, N, T)
                peak = torch.cuda.max_memory_allocated(dev)
            del T
            free()
            tried.append({"N": N, "ok": r is not None, "ms": r and r["ms"], "why": why})
            if r is None:
                fail_n, fail_why = N, why
                break
            ok_n = N
            N *= 2
        # bisect the largest N whose tensors exist (allocation or the library's shape check)
        lo, hi = ok_n or 0, fail_n
        while hi - lo > 1024:
            mid = (lo + hi) // 2 // 1024 * 1024
            if mid <= lo:
                break
            T, why = alloc(impl, mid)
            good = T is not None
            del T
            free()
            lo, hi = (mid, hi) if good else (lo, mid)
        if impl == "ours" and fa.fa_bwd_workspace_bytes(B, H, hi - 1, d) != 0:
            lo = hi - 1  # the library's limit is exact: the last N it accepts
        # run the step at the largest N that allocates (stepping down if the call itself fails)
        best, best_rec = None, None
        n_try = lo
        while n_try >= (ok_n or 0) and n_try > 0:
            T, why = alloc(impl, n_try)
            if T is not None:
                torch.cuda.reset_peak_memory_stats(dev)
                r, why = run(impl, n_try, T)
                peak = torch.cuda.max_memory_allocated(dev)
            else:
                r = None
            del T
            free()
            tried.append({"N": n_try, "ok": r is not None, "ms": r and r["ms"], "why": why})
            if r is not None:
                best, best_rec = n_try, {**r, "peak_hbm_bytes": peak}
                break
            n_try -= 1024
        flops = 14.0 * B * H * best * best * d / 2 if best else 0.0  # fwd + bwd, causal
        line = {"probe": "max_n", "impl": impl, "B": B, "H": H, "d": d, "causal": True,
                "step": ("fa_fwd (with the residual) + fa_bwd" if impl == "ours" else
                         "standard attention fwd + bwd (S fp32, P bf16 in HBM)"),
                "max_n_run": best, "step_ms": best_rec and best_rec["ms"],
                "step_tflops": (flops / (best_rec["ms"] / 1e3) / 1e12) if best_rec else None,
                "peak_hbm_bytes": best_rec and best_rec["peak_hbm_bytes"], "device_memory_bytes": total,
                "outputs_finite": best_rec and best_rec["finite"],
                "first_failure": {"N": fail_n, "why": fail_why}, "tried": tried}
        print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse_args()
    world, rank, local = dist_setup()
    from io_aware_exact_23_b200.inputs import CONFIGS
    if args.sweep:
        return run_sweep(args)
    if args.max_n:
        return run_max_n(args)
    w = CONFIGS[args.workload]
    if args.fp8:
        return run_fp8(args, w)
    if args.impl == "reference":
        return run_reference(args, w, world, rank)
    if args.impl == "vanilla":
        return run_vanilla(args, w)
    if args.dropout > 0.0 and args.deterministic:
        raise SystemExit("bench.py: --dropout and --deterministic are separate arms")
    if args.dropout > 0.0 or args.deterministic:
        return run_variant(args, w)

    import torch
    import torch.distributed as dist
    if not torch.cuda.is_available():
        raise SystemExit("bench.py: no CUDA device (the attention path has no CPU fallback)")
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    from io_aware_exact_23_b200 import binding as fa
    from io_aware_exact_23_b200.inputs import make_inputs, score_matrix_bytes

    dev = torch.device("cuda", local)
    t = make_inputs(rank_workload(w, rank), device=dev)
    q, k, v, dO = t["q"], t["k"], t["v"], t["do"]
    B, H, N, d = q.shape
    o = torch.empty_like(q)
    o_lo = torch.empty_like(q)  # O's rounding residual: exact D in the backward
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    ws = torch.empty(fa.fa_bwd_workspace_bytes(B, H, N, d), dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()
    torch.cuda.reset_peak_memory_stats(dev)

    def step(ev_f=None, ev_b=None):
        if ev_f is not None:
            ev_f[0].record()
        fa.fa_fwd(q, k, v, o, lse, w.scale, w.causal, o_lo=o_lo)
        if ev_f is not None:
            ev_f[1].record()
        fa.fa_bwd(q, k, v, o, dO, lse, dq, dk, dv, w.scale, w.causal, ws, events=ev_b, o_lo=o_lo)

    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize()
    if fa.fa_device_status() != 0:
        raise SystemExit("bench.py: device status error during warm-up")

    K = args.steps
    mk = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    ev_f = [(mk(), mk()) for _ in range(K)]
    ev_b = [tuple(mk() for _ in range(4)) for _ in range(K)]
    start, end = mk(), mk()
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    sampler = ClockSampler(uuid)
    sampler.wait_ready()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    tw0 = time.time()
    start.record()
    for s in range(K):
        step(ev_f[s], ev_b[s])
    end.record()
    torch.cuda.synchronize()
    tw1 = time.time()
    if world > 1:
        dist.barrier()
    sampler.stop()
    status = fa.fa_device_status()
    ms = start.elapsed_time(end)
    fwd_ms = statistics.mean(a.elapsed_time(b) for a, b in ev_f)
    pre_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev_b)
    main_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev_b)
    conv_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in ev_b)
    bwd_ms = statistics.mean(e[0].elapsed_time(e[3]) for e in ev_b)
    peak_mem = torch.cuda.max_memory_allocated(dev)  # inputs + outputs + workspace
    ms, fwd_ms, bwd_ms, main_ms, pre_ms, conv_ms, status = reduce_max(
        [ms, fwd_ms, bwd_ms, main_ms, pre_ms, conv_ms, float(status)], dist, dev)

    # ---------------------------------------------------------------- e2e
    # The same step from pinned host memory and back, every step: copy the step's
    # Q, K, V, dO in, run fa_fwd + fa_bwd through the C ABI, copy O, LSE, dQ, dK,
    # dV out.  Two device buffer sets and three streams (copy-in, compute,
    # copy-out) ordered by events let step t's compute overlap step t+1's
    # inputs and step t-1's outputs; every step's copies are inside the timed
    # region, which ends when the last step's outputs have reached the host.
    e2e = None
    if args.e2e_steps > 0:
        names_in, names_out = ("q", "k", "v", "do"), ("o", "lse", "dq", "dk", "dv")
        pin = {nm: t[nm].cpu().pin_memory() for nm in names_in}
        dev_sets = [{"q": q, "k": k, "v": v, "do": dO, "o": o, "o_lo": o_lo, "lse": lse, "dq": dq, "dk": dk,
                     "dv": dv, "ws": ws}]
        dev_sets.append({nm: torch.empty_like(x) for nm, x in dev_sets[0].items()})
        host_out = [{nm: torch.empty(dev_sets[0][nm].shape, dtype=dev_sets[0][nm].dtype, pin_memory=True)
                     for nm in names_out} for _ in range(2)]
        h2d = sum(x.numel() * x.element_size() for x in pin.values())
        d2h = sum(x.numel() * x.element_size() for x in host_out[0].values())
        s_in, s_comp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        E = args.e2e_steps
        ev_in = [torch.cuda.Event() for _ in range(E)]
        ev_comp = [torch.cuda.Event() for _ in range(E)]
        ev_out = [torch.cuda.Event() for _ in range(E)]
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0, e1 = mk(), mk()
        e0.record(s_in)
        for st in range(E):
            D, Hh = dev_sets[st % 2], host_out[st % 2]
            with torch.cuda.stream(s_in):
                if st >= 2:
                    s_in.wait_event(ev_comp[st - 2])  # set st % 2's inputs were consumed
                for nm in names_in:
                    D[nm].copy_(pin[nm], non_blocking=True)
                ev_in[st].record(s_in)
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(ev_in[st])
                if st >= 2:
                    s_comp.wait_event(ev_out[st - 2])  # set st % 2's outputs reached the host
                fa.fa_fwd(D["q"], D["k"], D["v"], D["o"], D["lse"], w.scale, w.causal, o_lo=D["o_lo"])
                fa.fa_bwd(D["q"], D["k"], D["v"], D["o"], D["do"], D["lse"], D["dq"], D["dk"], D["dv"], w.scale,
                          w.causal, D["ws"], o_lo=D["o_lo"])
                ev_comp[st].record(s_comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[st])
                for nm in names_out:
                    Hh[nm].copy_(D[nm], non_blocking=True)
                ev_out[st].record(s_out)
        s_in.wait_stream(s_out)
        e1.record(s_in)
        torch.cuda.synchronize()
        if fa.fa_device_status() != 0:
            raise SystemExit("bench.py: device status error in the e2e leg")
        e2e_ms = reduce_max([e0.elapsed_time(e1) / E], dist, dev)[0]
        # The host link's floor for the same bytes: the same copies, both directions
        # at once on their two streams, with no kernels between them.
        torch.cuda.synchronize()
        c0, c1 = mk(), mk()
        c0.record(s_in)
        s_out.wait_stream(s_in)
        for st in range(E):
            D, Hh = dev_sets[st % 2], host_out[st % 2]
            with torch.cuda.stream(s_in):
                for nm in names_in:
                    D[nm].copy_(pin[nm], non_blocking=True)
            with torch.cuda.stream(s_out):
                for nm in names_out:
                    Hh[nm].copy_(D[nm], non_blocking=True)
        s_in.wait_stream(s_out)
        c1.record(s_in)
        torch.cuda.synchronize()
        copy_ms = reduce_max([c0.elapsed_time(c1) / E], dist, dev)[0]
        e2e = {"value": world * (w.fwd_flops() + w.bwd_flops()) / (e2e_ms / 1e3) / 1e12, "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": E,
               "copies_alone_ms_per_step": copy_ms, "copy_floor_frac": copy_ms / e2e_ms,
               "path": "pinned host -> device copies, fa_fwd + fa_bwd through the C ABI, outputs -> pinned host; "
                       "two buffer sets, copy-in / compute / copy-out streams overlapped across steps"}

    if rank == 0:
        peaks, peak_kind = load_peaks()
        flops_step = w.fwd_flops() + w.bwd_flops()
        value = world * flops_step * K / (ms / 1e3) / 1e12
        fwd_tf = w.fwd_flops() / (fwd_ms / 1e3) / 1e12
        bwd_tf = w.bwd_flops() / (bwd_ms / 1e3) / 1e12
        main_tf = w.bwd_flops() / (main_ms / 1e3) / 1e12
        peak = float(peaks["bf16_tflops"])
        peak_sus = float(peaks.get("bf16_tflops_sustained", peak))
        kernels = {"fa_fwd_kernel": fwd_ms, "fa_bwd_pre_kernel": pre_ms, "fa_bwd_kernel": main_ms,
                   "fa_dq_convert_kernel": conv_ms}
        dominant = max(kernels, key=kernels.get)
        dom_flops = w.bwd_flops() if dominant in ("fa_bwd_kernel",) else (
            w.fwd_flops() if dominant == "fa_fwd_kernel" else 0.0)
        dom_tf = dom_flops / (kernels[dominant] / 1e3) / 1e12
        clocks = sampler.summary(tw0, tw1)
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_step": ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "B": B, "H": H, "N": N, "d": d, "causal": w.causal,
                       "per_rank": "the full workload on every rank (independent heads, no collective)",
                       "l2": l2_note(w)},
            "fwd_tflops": fwd_tf, "bwd_tflops": bwd_tf,
            "fwd_frac_of_peak": fwd_tf / peak, "bwd_frac_of_peak": bwd_tf / peak,
            "kernel_ms": kernels,
            "roofline": {"bound": "tensor", "kernel": dominant, "achieved": dom_tf, "peak": peak,
                         "unit": "TFLOP/s", "frac": dom_tf / peak,
                         "peak_kind": f"bf16 dense, burst, {peak_kind} (MEASURED_PEAKS.json)",
                         "frac_of_sustained": dom_tf / peak_sus,
                         "traffic": stored_traffic(dominant, w.name)},
            "peak_hbm_bytes": peak_mem,
            # libfa.so's device image, resident on every GPU that loads it, outside
            # torch's allocator: the no-alloc backward's static scratch array plus
            # its status word (and the 32-byte allocated status block).
            "library_resident_bytes": fa.NOALLOC_SCRATCH_BYTES + 32 + 32,
            "score_matrix_bytes_bf16": score_matrix_bytes(B, H, N, 2),
            "clocks": clocks,
            "gpu_launches": 4 * K,
            "device_status": int(status),
        }
        if e2e is not None:
            line["e2e"] = e2e
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline_sample(w, args.cpu_budget_s)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
