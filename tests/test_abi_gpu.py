"""The plain entry points of include/fa.h on the GPU, called through ctypes with raw device
pointers exactly as a C caller would: fa_fwd(q, k, v, o, lse, B, H, N, d, scale, causal,
stream) and fa_bwd(..., workspace, workspace_bytes, ...) (the flash_attn_func-style
interface of the holysheep.ai review, "Implementing Flash Attention in Your Architecture"),
checked against the fp64 oracle.  Also: a call that returns an error enqueues nothing on
its stream, and first calls made from several host threads at once all succeed."""
import ctypes
import os
import subprocess
import sys
import textwrap

import pytest
import torch

from exact_io_aware_93_b200 import api
from exact_io_aware_93_b200.inputs import WORKLOADS, make_inputs
from tests.parity import GRAD_TOL, LSE_TOL, O_TOL, fwd_errors, grad_errors

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
vp, ci, cf = ctypes.c_void_p, ctypes.c_int, ctypes.c_float


def _plain():
    L = api.lib()
    L.fa_fwd.argtypes = [vp] * 5 + [ci] * 4 + [cf, ci, vp]
    L.fa_fwd.restype = ci
    L.fa_bwd.argtypes = [vp] * 10 + [ctypes.c_size_t] + [ci] * 4 + [cf, ci, vp]
    L.fa_bwd.restype = ci
    L.fa_bwd_workspace_size.argtypes = [ci] * 4
    L.fa_bwd_workspace_size.restype = ctypes.c_size_t
    return L


def _stream():
    return vp(torch.cuda.current_stream().cuda_stream)


def _fwd(L, t, B, H, N, d, scale, causal, stream=None):
    return L.fa_fwd(t["q"].data_ptr(), t["k"].data_ptr(), t["v"].data_ptr(), t["o"].data_ptr(),
                    t["lse"].data_ptr(), B, H, N, d, cf(scale), int(causal), stream or _stream())


def _bwd(L, t, ws, ws_bytes, B, H, N, d, scale, causal, stream=None):
    return L.fa_bwd(t["q"].data_ptr(), t["k"].data_ptr(), t["v"].data_ptr(), t["o"].data_ptr(),
                    t["do"].data_ptr(), t["lse"].data_ptr(), t["dq"].data_ptr(), t["dk"].data_ptr(),
                    t["dv"].data_ptr(), ws, ws_bytes, B, H, N, d, cf(scale), int(causal), stream or _stream())


def _buffers(inp, B, H, N, d):
    t = {n: inp[n].cuda() for n in ("q", "k", "v", "do")}
    for n in ("o", "dq", "dk", "dv"):
        t[n] = torch.full_like(t["q"], float("nan"))
    t["lse"] = torch.full((B, H, N), float("nan"), dtype=torch.float32, device="cuda")
    return t


def test_plain_fwd_bwd_on_the_b4_h16_n2048_shape():
    """fa_fwd then fa_bwd at B=4, H=16, N=2048, d=128, causal: O and LSE of every row of
    four heads, dQ/dK/dV of two whole heads, against the oracle."""
    w = WORKLOADS["causal_b4_h16_n2048_d128"]
    B, H, N, d = w.B, w.H, w.N, w.d
    inp = make_inputs(B, H, N, d, w.seed, with_do=True)   # the workload's Q, K, V, then dO
    L = _plain()
    t = _buffers(inp, B, H, N, d)
    assert _fwd(L, t, B, H, N, d, w.scale, True) == 0
    need = L.fa_bwd_workspace_size(B, H, N, d)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    assert _bwd(L, t, ws.data_ptr(), need, B, H, N, d, w.scale, True) == 0
    torch.cuda.synchronize()
    assert api.get_status() == 0
    heads = [(0, 0), (1, 5), (2, 10), (3, 15)]
    eo, el, where = fwd_errors(inp, t["o"], t["lse"], w.scale, True, heads=heads)
    assert eo <= O_TOL and el <= LSE_TOL, (eo, el, where)
    g = {n: t[n].cpu() for n in ("dq", "dk", "dv")}
    err = grad_errors(inp, g, w.scale, True, [(0, 3), (3, 12)], [])
    assert max(err.values()) <= GRAD_TOL, err


def _captured_nodes(fn):
    """Number of graph nodes `fn(stream)` enqueues, captured on a side stream."""
    from cuda.bindings import runtime as rt
    s = torch.cuda.Stream()
    sp = vp(s.cuda_stream)
    (err,) = rt.cudaStreamBeginCapture(s.cuda_stream, rt.cudaStreamCaptureMode.cudaStreamCaptureModeRelaxed)
    assert err == rt.cudaError_t.cudaSuccess
    rc = fn(sp)
    err, graph = rt.cudaStreamEndCapture(s.cuda_stream)
    assert err == rt.cudaError_t.cudaSuccess
    err, _, n = rt.cudaGraphGetNodes(graph, 0)
    assert err == rt.cudaError_t.cudaSuccess
    rt.cudaGraphDestroy(graph)
    return rc, n


def test_an_error_enqueues_nothing():
    B, H, N, d, scale = 1, 2, 300, 128, 128 ** -0.5
    L = _plain()
    t = _buffers(make_inputs(B, H, N, d, 5, with_do=True), B, H, N, d)
    need = L.fa_bwd_workspace_size(B, H, N, d)
    ws = torch.empty(need + 64, dtype=torch.uint8, device="cuda")
    # one good call of each first (outside capture), so every per-device set-up is done
    assert _fwd(L, t, B, H, N, d, scale, True) == 0
    assert _bwd(L, t, ws.data_ptr(), need, B, H, N, d, scale, True) == 0
    torch.cuda.synchronize()
    rc, n = _captured_nodes(lambda s: _bwd(L, t, ws.data_ptr(), need, B, H, N, d, scale, True, s))
    assert rc == 0 and n == 3                                            # pre, main, post
    rc, n = _captured_nodes(lambda s: _fwd(L, t, B, H, N, d, scale, True, s))
    assert rc == 0 and n == 1
    bad = [
        lambda s: _bwd(L, t, ws.data_ptr(), need - 16, B, H, N, d, scale, True, s),       # workspace
        lambda s: _bwd(L, t, ws.data_ptr() + 8, need, B, H, N, d, scale, True, s),        # alignment
        lambda s: _bwd(L, t, ws.data_ptr(), need, B, H, N, 96, scale, True, s),           # head dim
        lambda s: _bwd(L, t, ws.data_ptr(), need, B, H, N, d, -1.0, True, s),             # scale
        lambda s: _bwd(L, t, ws.data_ptr(), need, B, H, N, d, scale, 2, s),               # causal flag
        lambda s: _fwd(L, t, B, H, 0, d, scale, True, s),                                 # N
        lambda s: _fwd(L, t, B, H, N, 80, scale, False, s),                               # head dim
    ]
    for fn in bad:
        rc, n = _captured_nodes(fn)
        assert rc != 0 and n == 0, (rc, n)
    assert api.get_status() == 0


def test_first_calls_from_several_threads_at_once():
    """In a fresh process eight threads make the library's first call on the device at the
    same moment; all must succeed (the per-device set-up is serialised)."""
    code = textwrap.dedent(f"""
        import sys, threading, ctypes
        sys.path.insert(0, {ROOT!r})
        import torch
        from exact_io_aware_93_b200 import api
        from exact_io_aware_93_b200.inputs import make_inputs
        inp = make_inputs(1, 2, 256, 128, 3)
        q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
        L = api.lib()
        vp, ci, cf = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        L.fa_fwd.argtypes = [vp] * 5 + [ci] * 4 + [cf, ci, vp]
        L.fa_fwd.restype = ci
        outs = [(torch.empty_like(q), torch.empty(1, 2, 256, device="cuda")) for _ in range(8)]
        torch.cuda.synchronize()
        go = threading.Barrier(8)
        rcs = [None] * 8
        def work(i):
            torch.cuda.set_device(0)
            go.wait()
            rcs[i] = L.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), outs[i][0].data_ptr(),
                              outs[i][1].data_ptr(), 1, 2, 256, 128, cf(0.088), 1, None)
        th = [threading.Thread(target=work, args=(i,)) for i in range(8)]
        for x in th: x.start()
        for x in th: x.join()
        torch.cuda.synchronize()
        assert all(o.equal(outs[0][0]) for o, _ in outs), "results differ"
        print("rcs", rcs)
        sys.exit(0 if rcs == [0] * 8 else 1)
    """)
    res = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stdout + res.stderr
