"""Out-of-bounds writes, caught without a sanitizer: every buffer the library writes (O, LSE,
dQ, dK, dV, the backward and decode workspaces, the allocation-free entry point's outputs) is
placed inside a larger allocation whose guard zones before and after it hold a NaN bit
pattern, and after each call the guard zones must be bit-identical.  The calls go through
the C ABI with raw pointers into the middle of those allocations, on small and ragged
shapes (tails of 1, 7, 44 and 127 rows past a 128-row tile, grouped heads, windows, fp16,
e4m3, decoding with empty and partial caches)."""
import ctypes

import numpy as np
import pytest
import torch

from exact_io_aware_93_b200 import api
from exact_io_aware_93_b200.inputs import make_decode_inputs, make_inputs, make_inputs_e4m3

pytestmark = pytest.mark.gpu

GUARD = 4096                        # bytes on each side; keeps the payload 256-byte aligned
PATTERN = 0x7FC00A5A                # a quiet NaN with a payload no kernel writes
vp, ci, cf = ctypes.c_void_p, ctypes.c_int, ctypes.c_float


class Guarded:
    """`nbytes` of payload between two guard zones, all pre-filled with PATTERN."""

    def __init__(self, nbytes: int):
        self.nbytes = int(nbytes)
        total = GUARD + (self.nbytes + 3) // 4 * 4 + GUARD
        self.words = torch.full((total // 4,), PATTERN, dtype=torch.int64, device="cuda").to(torch.int32)
        self.buf = self.words.view(torch.uint8)
        self.ptr = self.buf.data_ptr() + GUARD

    def view(self, shape, dtype):
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        assert n <= self.nbytes
        return self.buf[GUARD:GUARD + n].view(dtype).view(shape)

    def guards_intact(self) -> bool:
        w = self.words.cpu().numpy().view(np.uint32)
        head = w[:GUARD // 4]
        tail = w[(GUARD + (self.nbytes + 3) // 4 * 4) // 4:]
        # the payload's last partial word (if any) is not checked; the zones are
        return bool((head == PATTERN).all() and (tail == PATTERN).all())


def _lib():
    return api.lib()


def _stream():
    return vp(torch.cuda.current_stream().cuda_stream)


def _status_ok():
    torch.cuda.synchronize()
    assert api.get_status() == 0


FWD_CASES = [  # B, H, H_kv, N, d, causal, window, dtype
    (1, 1, 1, 1, 64, False, -1, torch.bfloat16),
    (2, 3, 3, 7, 128, True, -1, torch.bfloat16),
    (1, 2, 2, 129, 64, True, -1, torch.bfloat16),
    (1, 4, 2, 300, 128, True, 17, torch.bfloat16),
    (2, 2, 1, 255, 128, False, -1, torch.float16),
    (1, 2, 2, 640, 128, True, 128, torch.float16),
]


@pytest.mark.parametrize("B,H,H_kv,N,d,causal,window,dtype", FWD_CASES)
def test_forward_and_backward_write_only_their_buffers(B, H, H_kv, N, d, causal, window, dtype):
    L = _lib()
    inp = make_inputs(B, H, N, d, seed=600 + N, with_do=True, H_kv=H_kv, dtype=dtype)
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "do"))
    p = api.FaProblem(B, H, H_kv, N, d, d ** -0.5, int(causal), window, api.FA_DTYPE[dtype])
    esz = 2
    g_o = Guarded(B * N * H * d * esz)
    g_lse = Guarded(B * H * N * 4)
    st = L.fa_fwd_ex(ctypes.byref(p), q.data_ptr(), k.data_ptr(), v.data_ptr(), g_o.ptr, g_lse.ptr, _stream())
    assert st == 0
    _status_ok()
    assert g_o.guards_intact() and g_lse.guards_intact()
    o = g_o.view((B, N, H, d), dtype)
    lse = g_lse.view((B, H, N), torch.float32)
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()   # every element written
    need = int(L.fa_bwd_workspace_size_ex(ctypes.byref(p)))
    g_ws = Guarded(need)
    g_dq = Guarded(B * N * H * d * esz)
    g_dk = Guarded(B * N * H_kv * d * esz)
    g_dv = Guarded(B * N * H_kv * d * esz)
    o_c, lse_c = o.clone(), lse.clone()
    st = L.fa_bwd_ex(ctypes.byref(p), q.data_ptr(), k.data_ptr(), v.data_ptr(), o_c.data_ptr(), do.data_ptr(),
                     lse_c.data_ptr(), g_dq.ptr, g_dk.ptr, g_dv.ptr, g_ws.ptr, need, _stream())
    assert st == 0
    _status_ok()
    for g in (g_ws, g_dq, g_dk, g_dv):
        assert g.guards_intact()
    for g, shape in ((g_dq, (B, N, H, d)), (g_dk, (B, N, H_kv, d)), (g_dv, (B, N, H_kv, d))):
        assert torch.isfinite(g.view(shape, dtype)).all()


def test_e4m3_forward_writes_only_its_buffers():
    L = _lib()
    B, H, N, d = 1, 2, 300, 128
    inp = make_inputs_e4m3(B, H, N, d, seed=77)
    codes = {n: inp[n] for n in ("q", "k", "v")}
    scales = {n: inp[n + "_descale"] for n in ("q", "k", "v")}
    p = api.FaProblem(B, H, H, N, d, d ** -0.5, 1, -1, api.FA_DTYPE[torch.float8_e4m3fn])
    g_o, g_lse = Guarded(B * N * H * d * 2), Guarded(B * H * N * 4)
    st = L.fa_fwd_e4m3_scaled(ctypes.byref(p), codes["q"].cuda().data_ptr(), codes["k"].cuda().data_ptr(),
                              codes["v"].cuda().data_ptr(), cf(scales["q"]), cf(scales["k"]), cf(scales["v"]),
                              g_o.ptr, g_lse.ptr, _stream())
    assert st == 0
    _status_ok()
    assert g_o.guards_intact() and g_lse.guards_intact()


@pytest.mark.parametrize("lengths,N_q,G", [([0, 1, 200, 129], 1, 4), ([5, 300], 3, 2), ([1000], 8, 8)])
def test_decode_writes_only_its_buffers(lengths, N_q, G):
    L = _lib()
    B, H_kv, N_kv, d = len(lengths), 2, 1024, 128
    H = G * H_kv
    inp = make_decode_inputs(B, H, H_kv, N_q, N_kv, d, seed=91, lengths=lengths, tail_nan=True)
    q, k, v, sl = (inp[n].cuda() for n in ("q", "k", "v", "seqlens"))
    p = api.FaDecodeProblem(B, H, H_kv, N_q, N_kv, d, d ** -0.5, 1, -1, 0)
    need = int(L.fa_decode_workspace_size(ctypes.byref(p)))
    g_ws, g_o, g_lse = Guarded(need), Guarded(B * N_q * H * d * 2), Guarded(B * H * N_q * 4)
    st = L.fa_decode(ctypes.byref(p), q.data_ptr(), k.data_ptr(), v.data_ptr(), sl.data_ptr(), g_o.ptr, g_lse.ptr,
                     g_ws.ptr, need, _stream())
    assert st == 0
    _status_ok()
    for g in (g_ws, g_o, g_lse):
        assert g.guards_intact()
    assert torch.isfinite(g_o.view((B, N_q, H, d), torch.bfloat16)).all()


def test_noalloc_backward_writes_only_its_outputs():
    L = _lib()
    fn = L.fa_bwd_noalloc
    fn.argtypes = [vp] * 9 + [ci, ci, ci, ci, cf, ci, vp]
    fn.restype = ci
    B, H, N, d = 1, 3, 383, 128
    inp = make_inputs(B, H, N, d, seed=12, with_do=True)
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = api.fwd(q, k, v, causal=True)
    gs = [Guarded(B * N * H * d * 2) for _ in range(3)]
    for _ in range(2):
        st = fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(), lse.data_ptr(),
                gs[0].ptr, gs[1].ptr, gs[2].ptr, B, H, N, d, cf(d ** -0.5), 1, _stream())
        assert st == 0
        _status_ok()
        assert all(g.guards_intact() for g in gs)
