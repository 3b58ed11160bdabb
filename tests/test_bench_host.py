"""Host-side checks of bench.py's own logic (no GPU): the L2 note, the clock
summary (samples inside the timed region, the fallback window, throttle
reasons) and the per-kernel source hash."""
from __future__ import annotations

import importlib.util
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def load_bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_l2_note_tracks_the_workload():
    b = load_bench()
    from io_aware_exact_23_b200.inputs import C3, TINY
    assert "268 MB" in b.l2_note(C3) and "no flush" in b.l2_note(C3)
    assert "< 126 MB" in b.l2_note(TINY)


def make_sampler(b, samples):
    """A ClockSampler fed with given samples (it never starts nvidia-smi)."""
    s = b.ClockSampler.__new__(b.ClockSampler)
    s.samples = list(samples)
    s.proc = None
    return s


ROW = "{sm}, 1965, 700.0, 0x0000000000000004, Not Active, Not Active, Not Active, {cap}"


def test_clock_summary_inside_the_region():
    b = load_bench()
    s = make_sampler(b, [(10.0, ROW.format(sm=1965, cap="Not Active")), (10.1, ROW.format(sm=1800, cap="Active")),
                         (10.2, ROW.format(sm=1810, cap="Active")), (99.0, ROW.format(sm=100, cap="Not Active"))])
    out = s.summary(10.05, 10.25)
    assert out["samples"] == 2 and out["sm_mhz"] == 1805.0 and out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"] and out["window"] == "timed region"


def test_clock_summary_falls_back_to_nearby_samples():
    b = load_bench()
    s = make_sampler(b, [(10.0, ROW.format(sm=1965, cap="Not Active")), (10.3, ROW.format(sm=1950, cap="Not Active"))])
    out = s.summary(10.05, 10.10)  # shorter than the sampling period
    assert out["samples"] == 2 and out["window"].startswith("timed region +-")
    assert make_sampler(b, []).summary(0.0, 1.0)["sm_mhz"] is None


def test_source_hash_is_per_kernel():
    b = load_bench()
    f, g = b.source_sha("fa_fwd_kernel"), b.source_sha("fa_bwd_kernel")
    assert re.fullmatch(r"[0-9a-f]{16}", f) and re.fullmatch(r"[0-9a-f]{16}", g) and f != g


def test_reference_arm_prints_the_contract_line():
    """bench.py --impl reference (the CPU oracle) prints one JSON line with the contract's keys."""
    import json
    import subprocess
    import sys
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny_b1h2n256d64", "--steps", "2", "--warmup", "1"],
                         capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["config"]["workload"] == "tiny_b1h2n256d64"


def test_variant_arms_are_exclusive_and_need_a_device():
    """--dropout and --deterministic are separate arms; without a GPU every
    device arm refuses loudly instead of falling back to the CPU."""
    import subprocess
    import sys
    import torch
    run = lambda *a: subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *a],  # noqa: E731
                                    capture_output=True, text=True, timeout=300, cwd=ROOT)
    both = run("--dropout", "0.1", "--deterministic", "--steps", "1", "--warmup", "1")
    assert both.returncode != 0 and "separate arms" in both.stderr
    if not torch.cuda.is_available():
        for args in (("--deterministic",), ("--dropout", "0.1"), ()):
            out = run(*args, "--steps", "1", "--warmup", "1", "--no-cpu-baseline")
            assert out.returncode != 0 and not out.stdout.strip().startswith("{"), args
