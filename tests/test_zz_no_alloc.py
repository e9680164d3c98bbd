"""fa_bwd_noalloc: the backward pass for callers that cannot allocate device memory.

It runs on a scratch array built into the library instead of a caller workspace.  Its
results must match fa_bwd's and the fp64 oracle's (the parity tests' gradient tolerance)
on consecutive calls, because the shared scratch keeps the previous call's contents, and
the calls must leave the device's free memory unchanged.  This file is collected last,
so that a failure here does not stop the other tests from running.
"""
import ctypes

import pytest
import torch

from exact_io_aware_93_b200 import api
from exact_io_aware_93_b200.inputs import make_inputs
from tests.parity import GRAD_TOL, grad_errors

pytestmark = pytest.mark.gpu

NOALLOC_MAX_BYTES = 64 << 20


def _noalloc_fn():
    L = api.lib()
    vp, i = ctypes.c_void_p, ctypes.c_int
    fn = L.fa_bwd_noalloc
    fn.argtypes = [vp] * 9 + [i, i, i, i, ctypes.c_float, i, vp]
    fn.restype = i
    return fn


def _call(fn, t, dq, dk, dv, B, H, N, d, scale, causal):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return fn(t["q"].data_ptr(), t["k"].data_ptr(), t["v"].data_ptr(), t["o"].data_ptr(),
              t["do"].data_ptr(), t["lse"].data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
              B, H, N, d, ctypes.c_float(scale), int(causal), stream)


@pytest.mark.parametrize("B,H,N,d,causal", [(1, 4, 1000, 128, True), (2, 3, 777, 64, False)])
def test_noalloc_matches_workspace_path_twice(B, H, N, d, causal):
    fn = _noalloc_fn()
    inp = make_inputs(B, H, N, d, seed=4321 + N, with_do=True)
    t = {n: inp[n].cuda() for n in ("q", "k", "v", "do")}
    scale = d ** -0.5
    t["o"], t["lse"] = api.fwd(t["q"], t["k"], t["v"], causal=causal)
    ref = api.bwd(t["q"], t["k"], t["v"], t["o"], t["do"], t["lse"], causal=causal)
    torch.cuda.synchronize()
    heads = [(b, h) for b in range(B) for h in range(H)]
    for _ in range(2):
        dq, dk, dv = (torch.full_like(t["q"], float("nan")) for _ in range(3))
        rc = _call(fn, t, dq, dk, dv, B, H, N, d, scale, causal)
        assert rc == 0, api.FA_STATUS.get(rc)
        torch.cuda.synchronize()
        assert api.get_status() == 0
        for got, want in zip((dq, dk, dv), ref):
            err = float((got.float() - want.float()).abs().max()) / float(want.float().abs().max())
            assert err <= GRAD_TOL, err
        err = grad_errors(inp, {"dq": dq.cpu(), "dk": dk.cpu(), "dv": dv.cpu()}, scale, causal, heads, [])
        assert max(err.values()) <= GRAD_TOL, err


def test_noalloc_leaves_free_device_memory_unchanged():
    fn = _noalloc_fn()
    B, H, N, d = 1, 2, 640, 128
    inp = make_inputs(B, H, N, d, seed=99, with_do=True)
    t = {n: inp[n].cuda() for n in ("q", "k", "v", "do")}
    t["o"], t["lse"] = api.fwd(t["q"], t["k"], t["v"], causal=True)
    dq, dk, dv = (torch.empty_like(t["q"]) for _ in range(3))
    assert _call(fn, t, dq, dk, dv, B, H, N, d, d ** -0.5, True) == 0   # first call: set-up
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        assert _call(fn, t, dq, dk, dv, B, H, N, d, d ** -0.5, True) == 0
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert api.get_status() == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    fn = _noalloc_fn()
    x = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    t = {n: x for n in ("q", "k", "v", "o", "do")}
    t["lse"] = torch.zeros(16, dtype=torch.float32, device="cuda")
    B, H, N, d = 1, 64, 2048, 128
    assert 4 * B * H * (N * d + 2 * N) > NOALLOC_MAX_BYTES
    rc = _call(fn, t, x, x, x, B, H, N, d, d ** -0.5, True)
    assert rc == 7
