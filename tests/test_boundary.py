"""Host-side tests of the C ABI (no GPU needed): the library loads, exports
every function include/fa.h declares, and rejects bad arguments with the
documented status codes before touching any device."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")


@pytest.fixture(scope="module")
def lib():
    from io_aware_exact_23_b200 import build
    build.build()
    from io_aware_exact_23_b200 import binding
    return binding.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_api():
    names = declared_functions()
    for want in ("fa_fwd", "fa_bwd", "fa_bwd_workspace_bytes", "fa_status_string", "fa_device_status"):
        assert want in names


def test_library_exports_every_declared_symbol(lib):
    for nm in declared_functions():
        assert hasattr(lib, nm), f"libfa.so does not export {nm}"


def test_status_strings_cover_every_code(lib):
    src = open(HEADER).read()
    codes = {int(v) for v in re.findall(r"FA_[A-Z_]+ = (\d+)", src)}
    assert codes == set(range(9))
    seen = set()
    for c in codes:
        s = lib.fa_status_string(c).decode()
        assert s and not s.startswith("unknown")
        seen.add(s)
    assert len(seen) == len(codes)
    assert lib.fa_status_string(99).decode().startswith("unknown")
    assert lib.fa_status_string(-1)


P = ctypes.c_void_p(4096)  # 16-byte aligned dummy pointer: never dereferenced on error paths


def fwd(lib, *, q=P, o=P, lse=P, B=1, H=2, N=256, d=64, scale=0.125, causal=0):
    return lib.fa_fwd(q, P, P, o, lse, B, H, N, d, scale, causal, None)


def bwd(lib, *, ws=P, ws_bytes=1 << 30, B=1, H=2, N=256, d=64, scale=0.125, causal=0, dq=P):
    return lib.fa_bwd(P, P, P, P, P, P, dq, P, P, B, H, N, d, scale, causal, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,code", [
    ({"q": None}, 1), ({"o": None}, 1), ({"lse": None}, 1),
    ({"B": 0}, 1), ({"H": -1}, 1), ({"N": 0}, 1),
    ({"scale": 0.0}, 1), ({"scale": -1.0}, 1), ({"scale": float("inf")}, 1), ({"scale": float("nan")}, 1),
    ({"causal": 2}, 1), ({"d": 96}, 2), ({"d": 256}, 2), ({"d": 0}, 2),
    ({"B": 1 << 16, "H": 1 << 10, "N": 1 << 10}, 2),
    ({"q": ctypes.c_void_p(4100)}, 3), ({"lse": ctypes.c_void_p(4104)}, 3),
])
def test_fwd_argument_errors(lib, kw, code):
    assert fwd(lib, **kw) == code


@pytest.mark.parametrize("kw,code", [
    ({"dq": None}, 1), ({"N": 0}, 1), ({"d": 80}, 2), ({"ws": None}, 4), ({"ws_bytes": 16}, 4),
    ({"ws": ctypes.c_void_p(4104)}, 3), ({"dq": ctypes.c_void_p(4098)}, 3),
])
def test_bwd_argument_errors(lib, kw, code):
    assert bwd(lib, **kw) == code


def test_valid_arguments_without_a_device(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    assert fwd(lib) == 5
    assert bwd(lib) == 5
    assert lib.fa_device_status(None) == 5


def test_workspace_formula(lib):
    f = lib.fa_bwd_workspace_bytes
    f.restype = ctypes.c_size_t
    for B, H, N, d in [(1, 1, 1, 64), (2, 32, 4096, 128), (1, 2, 300, 128), (4, 16, 2048, 64)]:
        npad = (N + 127) // 128 * 128
        want = 4 * B * H * (N * d + 2 * npad)
        want = (want + 255) // 256 * 256 + 256  # + the backward kernel's unit counter
        assert f(B, H, N, d) == want
    assert f(1, 1, 256, 96) == 0 and f(0, 1, 256, 64) == 0


def test_binding_rejects_wrong_tensors():
    import torch
    from io_aware_exact_23_b200 import binding
    q = torch.zeros(1, 1, 128, 64, dtype=torch.float32)
    with pytest.raises(TypeError):
        binding.fa_fwd(q, q, q, q, torch.zeros(1, 1, 128), 0.1, False)
    qb = q.to(torch.bfloat16)
    with pytest.raises(ValueError):  # CPU tensors are refused: there is no CPU path
        binding.fa_fwd(qb, qb, qb, qb, torch.zeros(1, 1, 128), 0.1, False)


def test_product_path_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "io_aware_exact_23_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, fn)).read()
                assert "import oracle" not in txt and "from oracle" not in txt, fn
                assert "ref_attn" not in txt, fn


def test_dropout_argument_errors(lib):
    import ctypes as C
    u64, u32 = C.c_ulonglong, C.c_uint
    lib.fa_fwd_dropout.argtypes = [C.c_void_p] * 6 + [C.c_int] * 4 + [C.c_float, C.c_int, C.c_float, u64, u32,
                                                                      C.c_void_p]
    lib.fa_dropout_mask.argtypes = [C.c_int] * 3 + [C.c_float, u64, u32, C.c_void_p, C.c_void_p]

    def fwd_d(rate, d=64):
        return lib.fa_fwd_dropout(P, P, P, P, None, P, 1, 2, 256, d, 0.125, 0, rate, 1, 0, None)
    assert fwd_d(-0.1) == 1 and fwd_d(1.0) == 1 and fwd_d(float("nan")) == 1
    assert fwd_d(0.1, d=96) == 2
    assert lib.fa_dropout_mask(1, 2, 64, 1.5, 1, 0, P, None) == 1
    assert lib.fa_dropout_mask(1, 2, 64, 0.5, 1, 0, None, None) == 1
    import torch
    if not torch.cuda.is_available():
        assert fwd_d(0.1) == 5 and lib.fa_dropout_mask(1, 2, 64, 0.5, 1, 0, P, None) == 5


@pytest.mark.parametrize("kw,code", [
    ({"dq": None}, 1), ({"N": 0}, 1), ({"scale": 0.0}, 1), ({"causal": 3}, 1), ({"d": 80}, 2),
    ({"ws": None}, 4), ({"ws_bytes": 16}, 4), ({"ws": ctypes.c_void_p(4104)}, 3),
    ({"dq": ctypes.c_void_p(4098)}, 3), ({"o_lo": ctypes.c_void_p(4100)}, 3),
])
def test_deterministic_bwd_argument_errors(lib, kw, code):
    args = dict(ws=P, ws_bytes=1 << 30, N=256, d=64, scale=0.125, causal=0, dq=P, o_lo=None)
    args.update(kw)
    rc = lib.fa_bwd_deterministic(P, P, P, P, args["o_lo"], P, P, args["dq"], P, P, 1, 2, args["N"], args["d"],
                                  args["scale"], args["causal"], args["ws"], args["ws_bytes"], None)
    assert rc == code


def test_deterministic_bwd_without_a_device(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    assert lib.fa_bwd_deterministic(P, P, P, P, None, P, P, P, P, P, 1, 2, 256, 64, 0.125, 1, P, 1 << 30,
                                    None) == 5


def test_version_encodes_major_minor_patch(lib):
    v = lib.fa_version()
    assert v >= 200  # 0.2.0 added fa_bwd_deterministic
    major, minor, patch = v // 10000, v // 100 % 100, v % 100
    assert (major, minor, patch) >= (0, 2, 0)


def test_selftest_without_a_device(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    assert lib.fa_selftest_timeout(None) == 5


def fwd_fp8(lib, *, q=P, dq=P, o=P, lse=P, B=1, H=2, N=256, d=128, scale=0.125, causal=0):
    return lib.fa_fwd_fp8(q, P, P, dq, P, P, o, lse, B, H, N, d, ctypes.c_float(scale), causal, None)


@pytest.mark.parametrize("kw,code", [
    ({"q": None}, 1), ({"dq": None}, 1), ({"o": None}, 1), ({"lse": None}, 1), ({"N": 0}, 1),
    ({"scale": 0.0}, 1), ({"causal": 3}, 1), ({"d": 64}, 2), ({"d": 96}, 2),
    ({"B": 1 << 16, "H": 1 << 10, "N": 1 << 10}, 2),
    ({"q": ctypes.c_void_p(4097)}, 3), ({"o": ctypes.c_void_p(4104)}, 3), ({"dq": ctypes.c_void_p(4098)}, 3),
])
def test_fp8_fwd_argument_errors(lib, kw, code):
    """e4m3 forward: d = 128 only; 16-byte aligned tensors, 4-byte aligned descale vectors."""
    lib.fa_fwd_fp8.argtypes = [ctypes.c_void_p] * 8 + [ctypes.c_int] * 4 + [ctypes.c_float, ctypes.c_int,
                                                                           ctypes.c_void_p]
    assert fwd_fp8(lib, **kw) == code


def test_noalloc_status_calls_without_a_device(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    info = (ctypes.c_int * 4)(9, 9, 9, 9)
    assert lib.fa_noalloc_device_status(None, info) == 5
    assert list(info) == [0, 0, 0, 0]
    assert lib.fa_noalloc_selftest_timeout(None) == 5


def test_element_limit_is_exact(lib):
    """Tensors of up to 2^31 - 1 elements are accepted; one more row is refused."""
    f = lib.fa_bwd_workspace_bytes
    f.restype = ctypes.c_size_t
    for B, H, d in [(1, 1, 128), (1, 16, 128), (2, 32, 64)]:
        n_max = (2 ** 31 - 1) // (B * H * d)
        assert f(B, H, n_max, d) > 0
        assert f(B, H, n_max + 1, d) == 0
        assert fwd(lib, B=B, H=H, N=n_max + 1, d=d) == 2
