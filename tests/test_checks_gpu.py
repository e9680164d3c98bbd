"""The checking build (libfa_b200_checks.so, compiled with FA_CHECKS): every kernel compares
its TMA coordinates and global indices with the extents of the tensors they address.  On
valid problems of every kind (forward, backward, grouped heads, windows, fp16, e4m3, decode,
allocation-free backward; ragged lengths) no check may fire and the results must equal the
release library's; and a check made to fail by construction must be reported."""
import ctypes

import pytest
import torch

from exact_io_aware_93_b200 import api
from exact_io_aware_93_b200 import build as fabuild
from exact_io_aware_93_b200.inputs import make_decode_inputs, make_inputs, make_inputs_e4m3

pytestmark = pytest.mark.gpu
vp, ci, cf = ctypes.c_void_p, ctypes.c_int, ctypes.c_float


@pytest.fixture(scope="module")
def chk():
    L = ctypes.CDLL(fabuild.CHECKS_LIB_PATH)
    L.fa_fwd_ex.argtypes = [ctypes.POINTER(api.FaProblem)] + [vp] * 6
    L.fa_bwd_ex.argtypes = [ctypes.POINTER(api.FaProblem)] + [vp] * 10 + [ctypes.c_size_t, vp]
    L.fa_bwd_workspace_size_ex.argtypes = [ctypes.POINTER(api.FaProblem)]
    L.fa_bwd_workspace_size_ex.restype = ctypes.c_size_t
    L.fa_fwd_e4m3_scaled.argtypes = [ctypes.POINTER(api.FaProblem), vp, vp, vp, cf, cf, cf, vp, vp, vp]
    L.fa_decode_workspace_size.argtypes = [ctypes.POINTER(api.FaDecodeProblem)]
    L.fa_decode_workspace_size.restype = ctypes.c_size_t
    L.fa_decode.argtypes = [ctypes.POINTER(api.FaDecodeProblem), vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
    L.fa_bwd_noalloc.argtypes = [vp] * 9 + [ci, ci, ci, ci, cf, ci, vp]
    L.fa_get_status.argtypes = [vp]
    L.fa_get_status_site.argtypes = [vp, ctypes.POINTER(ci)]
    L.fa_selftest_bounds.argtypes = [vp]
    assert L.fa_checks_enabled() == 1
    return L


def _st():
    return vp(torch.cuda.current_stream().cuda_stream)


def _status(L):
    torch.cuda.synchronize()
    return L.fa_get_status(_st())


def test_a_failing_check_is_reported(chk):
    assert chk.fa_selftest_bounds(_st()) == 0
    assert _status(chk) == 8          # FA_ERR_BOUNDS, read and cleared
    assert _status(chk) == 0
    assert chk.fa_selftest_bounds(_st()) == 0
    site = ci(0)
    torch.cuda.synchronize()
    assert chk.fa_get_status_site(_st(), ctypes.byref(site)) == 8
    assert site.value == 999          # the self-test's own check site


CASES = [  # B, H, H_kv, N, d, causal, window, dtype
    (1, 1, 1, 1, 64, False, -1, torch.bfloat16),
    (2, 3, 3, 7, 128, True, -1, torch.bfloat16),
    (1, 2, 2, 129, 64, True, -1, torch.bfloat16),
    (1, 4, 2, 300, 128, True, 17, torch.bfloat16),
    (2, 2, 1, 255, 128, False, -1, torch.float16),
    (1, 2, 2, 700, 128, True, 200, torch.bfloat16),
    (1, 2, 2, 1000, 128, True, -1, torch.float16),
]


@pytest.mark.parametrize("B,H,H_kv,N,d,causal,window,dtype", CASES)
def test_forward_and_backward_pass_every_check(chk, B, H, H_kv, N, d, causal, window, dtype):
    inp = make_inputs(B, H, N, d, seed=700 + N, with_do=True, H_kv=H_kv, dtype=dtype)
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "do"))
    w = None if window < 0 else window
    o_ref, lse_ref = api.fwd(q, k, v, causal=causal, window=w)
    dq_ref, dk_ref, dv_ref = api.bwd(q, k, v, o_ref, do, lse_ref, causal=causal, window=w)
    p = api.FaProblem(B, H, H_kv, N, d, d ** -0.5, int(causal), window, api.FA_DTYPE[dtype])
    o, lse = torch.empty_like(q), torch.empty(B, H, N, device="cuda")
    assert chk.fa_fwd_ex(ctypes.byref(p), q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                         _st()) == 0
    assert _status(chk) == 0
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)
    need = chk.fa_bwd_workspace_size_ex(ctypes.byref(p))
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    assert chk.fa_bwd_ex(ctypes.byref(p), q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(),
                         lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ws.data_ptr(), need, _st()) == 0
    assert _status(chk) == 0
    assert torch.equal(dk, dk_ref) and torch.equal(dv, dv_ref)
    # dQ is summed with atomics: equal up to the order of the additions
    err = float((dq.float() - dq_ref.float()).abs().max()) / max(float(dq_ref.float().abs().max()), 1e-6)
    assert err < 1e-2


def test_e4m3_forward_passes_every_check(chk):
    B, H, N, d = 1, 2, 300, 128
    inp = make_inputs_e4m3(B, H, N, d, seed=5)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    o_ref, lse_ref = api.fwd_e4m3(q, k, v, inp["q_descale"], inp["k_descale"], inp["v_descale"], causal=True)
    p = api.FaProblem(B, H, H, N, d, d ** -0.5, 1, -1, api.FA_DTYPE[torch.float8_e4m3fn])
    o, lse = torch.empty_like(o_ref), torch.empty_like(lse_ref)
    assert chk.fa_fwd_e4m3_scaled(ctypes.byref(p), q.data_ptr(), k.data_ptr(), v.data_ptr(), inp["q_descale"],
                                  inp["k_descale"], inp["v_descale"], o.data_ptr(), lse.data_ptr(), _st()) == 0
    assert _status(chk) == 0
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)


@pytest.mark.parametrize("lengths,N_q,G", [([0, 1, 200, 129], 1, 4), ([5, 300], 3, 2), ([1000, 64], 8, 8)])
def test_decode_passes_every_check(chk, lengths, N_q, G):
    B, H_kv, N_kv, d = len(lengths), 2, 1024, 128
    H = G * H_kv
    inp = make_decode_inputs(B, H, H_kv, N_q, N_kv, d, seed=17, lengths=lengths, tail_nan=True)
    q, k, v, sl = (inp[n].cuda() for n in ("q", "k", "v", "seqlens"))
    o_ref, lse_ref = api.decode(q, k, v, sl, causal=True)
    p = api.FaDecodeProblem(B, H, H_kv, N_q, N_kv, d, d ** -0.5, 1, -1, 0)
    need = chk.fa_decode_workspace_size(ctypes.byref(p))
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    o, lse = torch.empty_like(o_ref), torch.empty_like(lse_ref)
    assert chk.fa_decode(ctypes.byref(p), q.data_ptr(), k.data_ptr(), v.data_ptr(), sl.data_ptr(), o.data_ptr(),
                         lse.data_ptr(), ws.data_ptr(), need, _st()) == 0
    assert _status(chk) == 0
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)


def test_noalloc_backward_passes_every_check(chk):
    B, H, N, d = 1, 3, 383, 128
    inp = make_inputs(B, H, N, d, seed=23, with_do=True)
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = api.fwd(q, k, v, causal=True)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    for _ in range(2):
        assert chk.fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(),
                                  lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, N, d,
                                  cf(d ** -0.5), 1, _st()) == 0
        assert _status(chk) == 0
