"""Thin Python binding of the C ABI in ``include/fa.h`` (argument marshalling only).

Every step of the computation runs in ``libfa_b200.so``; this module checks
tensor shapes the way the ``validate_attention_inputs`` helper of the
holysheep.ai review does (section "Common Errors and Fixes", error 4: same
batch, heads and head_dim for Q, K, V; same sequence length for K and V),
allocates outputs with PyTorch and passes raw device pointers.  There is no
fallback: without the compiled library, a CUDA tensor or an sm_100 device the
call raises.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

from . import build as _build

_lib = None

FA_STATUS = {
    0: "FA_OK", 1: "FA_ERR_INVALID_ARG", 2: "FA_ERR_UNSUPPORTED", 3: "FA_ERR_ALIGNMENT",
    4: "FA_ERR_DEVICE", 5: "FA_ERR_LAUNCH", 6: "FA_ERR_TIMEOUT", 7: "FA_ERR_WORKSPACE", 8: "FA_ERR_BOUNDS",
}


FA_DTYPE = {torch.bfloat16: 0, torch.float16: 1, torch.float8_e4m3fn: 2}


class FaProblem(ctypes.Structure):
    """The ``fa_problem`` descriptor of include/fa.h."""
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("H_kv", ctypes.c_int), ("N", ctypes.c_int),
                ("d", ctypes.c_int), ("scale", ctypes.c_float), ("causal", ctypes.c_int),
                ("window", ctypes.c_int), ("dtype", ctypes.c_int)]


class FaDecodeProblem(ctypes.Structure):
    """The ``fa_decode_problem`` descriptor of include/fa.h."""
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("H_kv", ctypes.c_int), ("N_q", ctypes.c_int),
                ("N_kv", ctypes.c_int), ("d", ctypes.c_int), ("scale", ctypes.c_float),
                ("causal", ctypes.c_int), ("window", ctypes.c_int), ("dtype", ctypes.c_int)]


class FAError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = int(status)
        super().__init__(f"{what}: {FA_STATUS.get(int(status), 'FA_ERR_UNKNOWN')} ({int(status)})")


def library_path() -> str:
    """The release library, or the checking build (every kernel bounds-checks its TMA
    coordinates and global indices and reports FA_ERR_BOUNDS) when the environment sets
    FA_B200_CHECKS=1 before the first call."""
    return _build.CHECKS_LIB_PATH if os.environ.get("FA_B200_CHECKS") == "1" else _build.LIB_PATH


def lib() -> ctypes.CDLL:
    """The loaded ``libfa_b200.so`` (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path):
        raise FileNotFoundError(
            f"{path} is missing; build it with `python -m exact_io_aware_93_b200.build` "
            "(there is no non-CUDA fallback)")
    L = ctypes.CDLL(path)
    vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    L.fa_abi_version.restype = i
    L.fa_status_string.argtypes = [i]
    L.fa_status_string.restype = ctypes.c_char_p
    L.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, vp]
    L.fa_fwd.restype = i
    L.fa_get_status.argtypes = [vp]
    L.fa_get_status.restype = i
    L.fa_get_status_site.argtypes = [vp, ctypes.POINTER(ctypes.c_int)]
    L.fa_get_status_site.restype = i
    L.fa_selftest_wait_timeout.argtypes = [ctypes.c_uint, vp]
    L.fa_selftest_wait_timeout.restype = i
    L.fa_bwd_workspace_size.argtypes = [i, i, i, i]
    L.fa_bwd_workspace_size.restype = ctypes.c_size_t
    L.fa_fwd_ex.argtypes = [ctypes.POINTER(FaProblem), vp, vp, vp, vp, vp, vp]
    L.fa_fwd_ex.restype = i
    L.fa_bwd_ex.argtypes = [ctypes.POINTER(FaProblem), vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                            ctypes.c_size_t, vp]
    L.fa_bwd_ex.restype = i
    L.fa_bwd_workspace_size_ex.argtypes = [ctypes.POINTER(FaProblem)]
    L.fa_bwd_workspace_size_ex.restype = ctypes.c_size_t
    L.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t,
                         i, i, i, i, f, i, vp]
    L.fa_bwd.restype = i
    L.fa_fwd_e4m3_scaled.argtypes = [ctypes.POINTER(FaProblem), vp, vp, vp, f, f, f, vp, vp, vp]
    L.fa_fwd_e4m3_scaled.restype = i
    L.fa_decode_workspace_size.argtypes = [ctypes.POINTER(FaDecodeProblem)]
    L.fa_decode_workspace_size.restype = ctypes.c_size_t
    L.fa_decode.argtypes = [ctypes.POINTER(FaDecodeProblem), vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
    L.fa_decode.restype = i
    _lib = L
    return L


def _stream_ptr(t: torch.Tensor):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _on(t: torch.Tensor):
    """Make t's device current for a library call: the library takes its SM count, kernel
    set-up and status word from the current device, and launches on that device's stream."""
    return torch.cuda.device(t.device)


def validate_inputs(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor) -> None:
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{name} must be a torch.Tensor")
        if t.dim() != 4:
            raise ValueError(f"{name} must be [batch, seq_len, num_heads, head_dim], got {tuple(t.shape)}")
        if t.dtype not in FA_DTYPE:
            raise TypeError(f"{name} must be bfloat16, float16 or float8_e4m3fn, got {t.dtype}")
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor (no CPU path)")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if not (q.shape[0] == k.shape[0] == v.shape[0]):
        raise ValueError(f"batch size mismatch: {q.shape[0]}, {k.shape[0]}, {v.shape[0]}")
    if k.shape[2] != v.shape[2] or q.shape[2] % k.shape[2] != 0:
        raise ValueError(f"num heads mismatch: {q.shape[2]}, {k.shape[2]}, {v.shape[2]} (key/value heads "
                         "must match each other and divide the query heads)")
    if k.shape[1] != v.shape[1]:
        raise ValueError(f"key/value sequence length mismatch: {k.shape[1]}, {v.shape[1]}")
    if not (q.shape[3] == k.shape[3] == v.shape[3]):
        raise ValueError(f"head dim mismatch: {q.shape[3]}, {k.shape[3]}, {v.shape[3]}")
    if q.shape[1] != k.shape[1]:
        raise ValueError(f"query and key sequence lengths must match: {q.shape[1]}, {k.shape[1]}")
    if not (q.device == k.device == v.device):
        raise ValueError("q, k, v must be on the same device")
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError(f"q, k, v must share one dtype, got {q.dtype}, {k.dtype}, {v.dtype}")


def check_buffer(name: str, t: torch.Tensor, shape, dtype: torch.dtype, device: torch.device) -> None:
    """A caller-supplied output must match exactly: the library writes through its raw pointer,
    so a smaller or misplaced buffer would be written out of bounds."""
    if (not isinstance(t, torch.Tensor) or tuple(t.shape) != tuple(shape) or t.dtype != dtype
            or t.device != device or not t.is_contiguous()):
        raise ValueError(f"{name} must be a contiguous {dtype} tensor of shape {tuple(shape)} on {device}")


def check_scratch(name: str, t: torch.Tensor, device: torch.device) -> None:
    """A caller-supplied workspace: any dtype, contiguous, on the inputs' device (its byte size
    is checked by the library)."""
    if not isinstance(t, torch.Tensor) or t.device != device or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous tensor on {device}")


def problem(q: torch.Tensor, k: torch.Tensor, causal: bool, scale: float | None,
            window: int | None) -> FaProblem:
    B, N, H, d = q.shape
    return FaProblem(B, H, k.shape[2], N, d, 1.0 / math.sqrt(d) if scale is None else float(scale),
                     int(bool(causal)), -1 if window is None else int(window), FA_DTYPE[q.dtype])


def fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
        scale: float | None = None, out: torch.Tensor | None = None,
        lse: torch.Tensor | None = None, window: int | None = None):
    """(O [B, N, H, d] in q's dtype, LSE [B, H, N] fp32) of exact attention via ``fa_fwd_ex``.

    k and v may have fewer heads than q (grouped-query attention); ``window`` (causal only)
    limits query i to keys i - window .. i."""
    validate_inputs(q, k, v)
    B, N, H, d = q.shape
    out_dtype = torch.bfloat16 if q.dtype == torch.float8_e4m3fn else q.dtype
    if out is None:
        out = torch.empty(q.shape, dtype=out_dtype, device=q.device)
    check_buffer("out", out, q.shape, out_dtype, q.device)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    check_buffer("lse", lse, (B, H, N), torch.float32, q.device)
    p = problem(q, k, causal, scale, window)
    with _on(q):
        st = lib().fa_fwd_ex(ctypes.byref(p), q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                             lse.data_ptr(), _stream_ptr(q))
    if st != 0:
        raise FAError(st, "fa_fwd_ex")
    return out, lse


def fwd_e4m3(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, q_descale: float, k_descale: float,
             v_descale: float, causal: bool = False, scale: float | None = None, out: torch.Tensor | None = None,
             lse: torch.Tensor | None = None, window: int | None = None):
    """(O [B, N, H, d] bf16, LSE [B, H, N] fp32) of attention over the values ``codes * descale``
    of fp8 e4m3 inputs (torch.float8_e4m3fn), via ``fa_fwd_e4m3_scaled`` (d = 128)."""
    validate_inputs(q, k, v)
    if q.dtype != torch.float8_e4m3fn:
        raise TypeError("fwd_e4m3 takes float8_e4m3fn codes")
    B, N, H, d = q.shape
    out = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device) if out is None else out
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device) if lse is None else lse
    check_buffer("out", out, q.shape, torch.bfloat16, q.device)
    check_buffer("lse", lse, (B, H, N), torch.float32, q.device)
    p = problem(q, k, causal, scale, window)
    with _on(q):
        st = lib().fa_fwd_e4m3_scaled(ctypes.byref(p), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                      float(q_descale), float(k_descale), float(v_descale), out.data_ptr(),
                                      lse.data_ptr(), _stream_ptr(q))
    if st != 0:
        raise FAError(st, "fa_fwd_e4m3_scaled")
    return out, lse


def bwd_workspace_size(B: int, H: int, N: int, d: int) -> int:
    """Bytes of device workspace ``fa_bwd`` needs (fp32 dQ accumulator and row sums D)."""
    return int(lib().fa_bwd_workspace_size(B, H, N, d))


def bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor, do: torch.Tensor,
        lse: torch.Tensor, causal: bool = False, scale: float | None = None,
        dq: torch.Tensor | None = None, dk: torch.Tensor | None = None, dv: torch.Tensor | None = None,
        workspace: torch.Tensor | None = None, window: int | None = None):
    """(dQ, dK, dV) of L = sum(O * dO) via ``fa_bwd_ex`` (score tiles recomputed from LSE)."""
    validate_inputs(q, k, v)
    for name, t in (("o", o), ("do", do)):
        if t.shape != q.shape or t.dtype != q.dtype or not t.is_contiguous() or t.device != q.device:
            raise ValueError(f"{name} must be a contiguous tensor shaped like q, of q's dtype")
    B, N, H, d = q.shape
    check_buffer("lse", lse, (B, H, N), torch.float32, q.device)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    check_buffer("dq", dq, q.shape, q.dtype, q.device)
    check_buffer("dk", dk, k.shape, k.dtype, q.device)
    check_buffer("dv", dv, v.shape, v.dtype, q.device)
    p = problem(q, k, causal, scale, window)
    need = int(lib().fa_bwd_workspace_size_ex(ctypes.byref(p)))
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    check_scratch("workspace", workspace, q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    with _on(q):
        st = lib().fa_bwd_ex(ctypes.byref(p), q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                             do.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                             workspace.data_ptr(), ws_bytes, _stream_ptr(q))
    if st != 0:
        raise FAError(st, "fa_bwd_ex")
    return dq, dk, dv


def decode_problem(q: torch.Tensor, k_cache: torch.Tensor, causal: bool, scale: float | None,
                   window: int | None) -> FaDecodeProblem:
    B, n_q, H, d = q.shape
    return FaDecodeProblem(B, H, k_cache.shape[2], n_q, k_cache.shape[1], d,
                           1.0 / math.sqrt(d) if scale is None else float(scale), int(bool(causal)),
                           -1 if window is None else int(window), FA_DTYPE.get(q.dtype, -1))


def decode_workspace_size(q: torch.Tensor, k_cache: torch.Tensor, causal: bool = True,
                          window: int | None = None) -> int:
    """Bytes of device workspace ``fa_decode`` needs for these shapes on q's device (the split
    depends on that device's SM count)."""
    with _on(q):
        return int(lib().fa_decode_workspace_size(ctypes.byref(decode_problem(q, k_cache, causal, None, window))))


def decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
           seqlens: torch.Tensor | None = None, causal: bool = True, scale: float | None = None,
           out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
           workspace: torch.Tensor | None = None, window: int | None = None):
    """(O [B, N_q, H, d] in q's dtype, LSE [B, H, N_q] fp32) of N_q new queries per sequence against a
    key/value cache ``[B, N_kv, H_kv, d]`` via ``fa_decode``.

    ``seqlens`` (int32 [B] on the device, or None for full caches) gives each sequence's cached
    length; with ``causal`` the queries are the last N_q positions of each sequence: query i
    of sequence b stands at position seqlens[b] - N_q + i."""
    for name, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache)):
        if not isinstance(t, torch.Tensor) or t.dim() != 4 or t.dtype not in FA_DTYPE or t.dtype != q.dtype:
            raise ValueError(f"{name} must be a 4-d bfloat16 or float16 tensor of q's dtype")
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor (no CPU path)")
    B, n_q, H, d = q.shape
    if k_cache.shape != v_cache.shape or k_cache.shape[0] != B or k_cache.shape[3] != d:
        raise ValueError(f"cache shapes {tuple(k_cache.shape)}, {tuple(v_cache.shape)} do not fit q {tuple(q.shape)}")
    if H % k_cache.shape[2] != 0:
        raise ValueError("key/value heads must divide the query heads")
    if not (k_cache.device == v_cache.device == q.device):
        raise ValueError("q, k_cache and v_cache must be on the same device")
    if seqlens is not None:
        check_buffer("seqlens", seqlens, (B,), torch.int32, q.device)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, H, n_q), dtype=torch.float32, device=q.device) if lse is None else lse
    check_buffer("out", out, q.shape, q.dtype, q.device)
    check_buffer("lse", lse, (B, H, n_q), torch.float32, q.device)
    p = decode_problem(q, k_cache, causal, scale, window)
    with _on(q):
        need = int(lib().fa_decode_workspace_size(ctypes.byref(p)))
        if workspace is None:
            workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
        check_scratch("workspace", workspace, q.device)
        ws_bytes = workspace.numel() * workspace.element_size()
        st = lib().fa_decode(ctypes.byref(p), q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                             None if seqlens is None else seqlens.data_ptr(), out.data_ptr(), lse.data_ptr(),
                             workspace.data_ptr(), ws_bytes, _stream_ptr(q))
    if st != 0:
        raise FAError(st, "fa_decode")
    return out, lse


def get_status(device: torch.device | None = None) -> int:
    """Synchronise the device's current stream and read-and-clear that device's status word
    (the current device when none is given)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        s = torch.cuda.current_stream(dev)
        return int(lib().fa_get_status(ctypes.c_void_p(s.cuda_stream)))


def get_status_site(device: torch.device | None = None) -> tuple[int, int]:
    """As get_status, and also where the first recorded error arose: the site number of the
    wait that ran out or of the bounds check that failed (0 when none was recorded)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    site = ctypes.c_int(0)
    with torch.cuda.device(dev):
        s = torch.cuda.current_stream(dev)
        st = int(lib().fa_get_status_site(ctypes.c_void_p(s.cuda_stream), ctypes.byref(site)))
    return st, int(site.value)


def selftest_wait_timeout(timeout_us: int = 20000) -> int:
    """Run the bounded-wait self-test on the current stream; returns the launch status."""
    s = torch.cuda.current_stream()
    return int(lib().fa_selftest_wait_timeout(int(timeout_us), ctypes.c_void_p(s.cuda_stream)))


def attention(q, k, v, causal: bool = False, scale: float | None = None) -> torch.Tensor:
    """O only."""
    return fwd(q, k, v, causal=causal, scale=scale)[0]
