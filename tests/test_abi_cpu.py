"""The C ABI library: builds, loads and exports every declared symbol; host-side
argument validation returns the documented codes without touching a GPU."""
import ctypes
import os
import re

import pytest

from exact_io_aware_93_b200 import build as fabuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in sorted(os.listdir(os.path.join(ROOT, "include")))
           if f.endswith(".h")]


def declared_functions():
    names = []
    for path in HEADERS:
        text = open(path).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        for m in re.finditer(r"^\s*[A-Za-z_][\w\s\*]*?\b(fa_\w+)\s*\(", text, flags=re.M):
            names.append(m.group(1))
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    path = fabuild.build()
    return ctypes.CDLL(path)


def test_headers_declare_entry_points():
    names = declared_functions()
    assert "fa_fwd" in names and "fa_get_status" in names and "fa_status_string" in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in include/*.h but not exported"


def test_status_strings(lib):
    lib.fa_status_string.restype = ctypes.c_char_p
    lib.fa_status_string.argtypes = [ctypes.c_int]
    assert lib.fa_status_string(0) == b"FA_OK"
    assert lib.fa_status_string(6) == b"FA_ERR_TIMEOUT"
    assert lib.fa_status_string(99) == b"FA_ERR_UNKNOWN"
    assert lib.fa_status_string(8) == b"FA_ERR_BOUNDS"
    assert lib.fa_abi_version() == 6


def _fwd(lib, q=0x10000, k=0x10000, v=0x10000, o=0x10000, lse=0x10000, B=1, H=1, N=16, d=64,
         scale=0.125, causal=0):
    vp = ctypes.c_void_p
    lib.fa_fwd.argtypes = [vp, vp, vp, vp, vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                           ctypes.c_float, ctypes.c_int, vp]
    lib.fa_fwd.restype = ctypes.c_int
    return lib.fa_fwd(vp(q), vp(k), vp(v), vp(o), vp(lse), B, H, N, d, ctypes.c_float(scale), causal, None)


def test_fwd_validation_codes(lib):
    assert _fwd(lib, q=0) == 1
    assert _fwd(lib, lse=0) == 1
    assert _fwd(lib, B=0) == 1
    assert _fwd(lib, N=0) == 1
    assert _fwd(lib, H=-1) == 1
    assert _fwd(lib, scale=0.0) == 1
    assert _fwd(lib, scale=float("nan")) == 1
    assert _fwd(lib, scale=float("inf")) == 1
    assert _fwd(lib, causal=2) == 1
    assert _fwd(lib, d=96) == 2
    assert _fwd(lib, d=256) == 2
    assert _fwd(lib, q=0x10008) == 3
    assert _fwd(lib, o=0x10004) == 3
    assert _fwd(lib, lse=0x10002) == 3
    assert _fwd(lib, B=1 << 20, H=1 << 10, N=1 << 20, d=128) == 1


def test_fwd_without_gpu_reports_device(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is visible: the device check passes")
    assert _fwd(lib) == 4


def test_bwd_validation_codes(lib):
    vp = ctypes.c_void_p
    lib.fa_bwd.argtypes = [vp] * 10 + [ctypes.c_size_t] + [ctypes.c_int] * 4 + [ctypes.c_float, ctypes.c_int, vp]
    lib.fa_bwd.restype = ctypes.c_int
    lib.fa_bwd_workspace_size.argtypes = [ctypes.c_int] * 4
    lib.fa_bwd_workspace_size.restype = ctypes.c_size_t
    ws = lib.fa_bwd_workspace_size(1, 1, 16, 64)
    assert ws == 4 * (16 * 64 + 2 * 128)
    assert lib.fa_bwd_workspace_size(1, 1, 16, 96) == 0
    # beyond the index range fa_bwd accepts: 0, not a wrapped-around byte count
    assert lib.fa_bwd_workspace_size(2**31 - 1, 2**31 - 1, 2**31 - 1, 128) == 0

    def call(p=0x10000, wsp=0x10000, wsb=ws, d=64, B=1, scale=0.125):
        return lib.fa_bwd(vp(p), vp(0x10000), vp(0x10000), vp(0x10000), vp(0x10000), vp(0x10000),
                          vp(0x10000), vp(0x10000), vp(0x10000), vp(wsp), wsb, B, 1, 16, d,
                          ctypes.c_float(scale), 0, None)
    assert call(p=0) == 1
    assert call(B=0) == 1
    assert call(scale=-1.0) == 1
    assert call(d=80) == 2
    assert call(p=0x10001) == 3
    assert call(wsp=0) == 7
    assert call(wsb=ws - 1) == 7
    assert call(wsp=0x10004) == 3


def test_selftest_validation_without_gpu(lib):
    lib.fa_selftest_wait_timeout.argtypes = [ctypes.c_uint, ctypes.c_void_p]
    lib.fa_selftest_wait_timeout.restype = ctypes.c_int
    assert lib.fa_selftest_wait_timeout(0, None) == 1
    assert lib.fa_selftest_wait_timeout(5_000_000, None) == 1


def test_ex_validation_codes(lib):
    from exact_io_aware_93_b200.api import FaProblem
    vp = ctypes.c_void_p
    lib.fa_fwd_ex.argtypes = [ctypes.POINTER(FaProblem), vp, vp, vp, vp, vp, vp]
    lib.fa_fwd_ex.restype = ctypes.c_int
    lib.fa_bwd_workspace_size_ex.argtypes = [ctypes.POINTER(FaProblem)]
    lib.fa_bwd_workspace_size_ex.restype = ctypes.c_size_t
    P = 0x10000

    def fwd(**kw):
        base = dict(B=1, H=4, H_kv=2, N=64, d=64, scale=0.125, causal=1, window=-1)
        base.update(kw)
        p = FaProblem(**base)
        return lib.fa_fwd_ex(ctypes.byref(p), vp(P), vp(P), vp(P), vp(P), vp(P), None)
    assert lib.fa_fwd_ex(None, vp(P), vp(P), vp(P), vp(P), vp(P), None) == 1
    assert fwd(H_kv=3) == 1          # does not divide H
    assert fwd(H_kv=0) == 1
    assert fwd(H_kv=8) == 1          # more key/value heads than query heads
    assert fwd(window=-2) == 1
    assert fwd(window=5, causal=0) == 1
    assert fwd(d=96) == 2
    assert fwd(dtype=3) == 2 and fwd(dtype=-1) == 2   # bf16 (0), fp16 (1), e4m3 (2)
    assert fwd(dtype=2, d=64) == 2                      # e4m3 is built for d = 128 only
    p = FaProblem(2, 4, 1, 100, 128, 0.1, 1, 16)
    assert lib.fa_bwd_workspace_size_ex(ctypes.byref(p)) == 4 * 2 * 4 * (100 * 128 + 2 * 128)


def test_decode_validation_codes(lib):
    """fa_decode checks its problem and pointers on the host, before any device work."""
    from exact_io_aware_93_b200.api import FaDecodeProblem
    vp = ctypes.c_void_p
    lib.fa_decode.argtypes = [ctypes.POINTER(FaDecodeProblem), vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
    lib.fa_decode.restype = ctypes.c_int
    lib.fa_decode_workspace_size.argtypes = [ctypes.POINTER(FaDecodeProblem)]
    lib.fa_decode_workspace_size.restype = ctypes.c_size_t
    P = 0x10000

    def dec(seqlens=None, q=P, lse=P, **kw):
        base = dict(B=2, H=8, H_kv=2, N_q=1, N_kv=1000, d=128, scale=0.1, causal=1, window=-1)
        base.update(kw)
        p = FaDecodeProblem(**base)
        return lib.fa_decode(ctypes.byref(p), vp(q), vp(P), vp(P), None if seqlens is None else vp(seqlens),
                             vp(P), vp(lse), vp(P), 1 << 30, None)
    assert lib.fa_decode(None, vp(P), vp(P), vp(P), None, vp(P), vp(P), vp(P), 0, None) == 1
    assert dec(q=0) == 1
    assert dec(B=0) == 1 and dec(N_q=0) == 1 and dec(N_kv=0) == 1
    assert dec(H_kv=3) == 1 and dec(H_kv=16) == 1
    assert dec(scale=0.0) == 1 and dec(causal=2) == 1
    assert dec(window=-2) == 1 and dec(window=4, causal=0) == 1
    assert dec(d=96) == 2
    assert dec(dtype=5) == 2
    assert dec(H=8, H_kv=1, N_q=17) == 2       # 8 heads x 17 positions > 128 rows
    assert dec(H=8, H_kv=1, N_q=16) != 2
    assert dec(q=P + 8) == 3
    assert dec(lse=P + 2) == 3
    assert dec(seqlens=P + 2) == 3
    import torch
    if not torch.cuda.is_available():
        assert dec() == 4                       # valid problem, no sm_100 device here
        p = FaDecodeProblem(2, 8, 2, 1, 1000, 128, 0.1, 1, -1)
        assert lib.fa_decode_workspace_size(ctypes.byref(p)) == 0


def test_e4m3_validation_codes(lib):
    from exact_io_aware_93_b200.api import FaProblem
    vp = ctypes.c_void_p
    f = ctypes.c_float
    lib.fa_fwd_e4m3_scaled.argtypes = [ctypes.POINTER(FaProblem), vp, vp, vp, f, f, f, vp, vp, vp]
    lib.fa_fwd_e4m3_scaled.restype = ctypes.c_int
    P = 0x10000

    def call(dtype=2, d=128, qd=1.0, kd=1.0, vd=1.0):
        p = FaProblem(1, 2, 2, 64, d, 0.1, 1, -1, dtype)
        return lib.fa_fwd_e4m3_scaled(ctypes.byref(p), vp(P), vp(P), vp(P), qd, kd, vd, vp(P), vp(P), None)
    assert lib.fa_fwd_e4m3_scaled(None, vp(P), vp(P), vp(P), 1.0, 1.0, 1.0, vp(P), vp(P), None) == 1
    assert call(dtype=0) == 1                 # this entry point is for e4m3 codes only
    assert call(d=64) == 2
    assert call(qd=0.0) == 1 and call(vd=float("inf")) == 1 and call(kd=-1.0) == 1
    import torch
    if not torch.cuda.is_available():
        assert call() == 4                    # valid, no sm_100 device here


def test_checking_build_exports_the_same_symbols_and_says_so(lib):
    chk = ctypes.CDLL(fabuild.CHECKS_LIB_PATH)
    for name in declared_functions():
        assert hasattr(chk, name), f"{name} declared in include/*.h but not exported by the checking build"
    assert lib.fa_checks_enabled() == 0
    assert chk.fa_checks_enabled() == 1
    # the release build has no checks: its self-test refuses before touching a device
    lib.fa_selftest_bounds.argtypes = [ctypes.c_void_p]
    assert lib.fa_selftest_bounds(None) == 2      # FA_ERR_UNSUPPORTED


def test_checking_build_keeps_the_register_contract():
    log = open(os.path.join(os.path.dirname(fabuild.CHECKS_LIB_PATH), "build_checks.log")).read()
    fabuild.check_register_contract(log)
