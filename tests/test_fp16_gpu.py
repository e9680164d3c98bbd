"""fp16 tensors through the forward, backward and decode entry points, against the fp64
oracle (the same definitions; only the input rounding differs)."""
import pytest
import torch

from exact_io_aware_93_b200 import api
from exact_io_aware_93_b200.inputs import EXTRA_WORKLOADS, make_decode_inputs, make_inputs, make_workload_inputs
from tests.parity import (GRAD_TOL, LSE_TOL, O_TOL, decode_errors, fwd_errors, fwd_errors_gqa, grad_errors,
                          grad_errors_gqa)

pytestmark = pytest.mark.gpu

CASES = [
    # B, H, H_kv, N, d, causal, window
    (1, 2, 2, 300, 128, True, -1),
    (2, 4, 4, 257, 64, False, -1),
    (1, 4, 2, 1000, 128, True, 100),
    (1, 3, 1, 129, 64, True, -1),
    (1, 2, 2, 1, 128, False, -1),
]


@pytest.mark.parametrize("B,H,Hkv,N,d,causal,window", CASES)
def test_fp16_fwd_bwd(B, H, Hkv, N, d, causal, window):
    inp = make_inputs(B, H, N, d, seed=9500 + N + H, with_do=True, H_kv=Hkv, dtype=torch.float16)
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "do"))
    w = None if window < 0 else window
    o, lse = api.fwd(q, k, v, causal=causal, window=w)
    dq, dk, dv = api.bwd(q, k, v, o, do, lse, causal=causal, window=w)
    torch.cuda.synchronize()
    assert api.get_status() == 0
    assert o.dtype == torch.float16 and dq.dtype == torch.float16 and dk.dtype == torch.float16
    eo, el = fwd_errors_gqa(inp, o, lse, d ** -0.5, causal, window)
    assert eo <= O_TOL and el <= LSE_TOL, (eo, el)
    err = grad_errors_gqa(inp, {"dq": dq.cpu(), "dk": dk.cpu(), "dv": dv.cpu()}, d ** -0.5, causal, window)
    assert max(err.values()) <= GRAD_TOL, err


def test_fp16_workload_sampled():
    """The forward + backward configuration with fp16 tensors, checked on sampled rows."""
    w = EXTRA_WORKLOADS["f16_causal_fwdbwd_b2_h16_n8192_d128"]
    inp = make_workload_inputs(w)
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = api.fwd(q, k, v, causal=True)
    dq, dk, dv = api.bwd(q, k, v, o, do, lse, causal=True)
    torch.cuda.synchronize()
    assert api.get_status() == 0
    heads = [(0, 0), (1, w.H - 1), (0, 7)]
    eo, el, where = fwd_errors(inp, o, lse, w.scale, True, rows_per_head=512, seed=w.seed, heads=heads)
    assert eo <= O_TOL and el <= LSE_TOL, (eo, el, where)
    import numpy as np
    rng = np.random.default_rng(w.seed)
    sampled = [(1, 5, np.sort(rng.choice(w.N, 256, replace=False))),
               (0, 11, np.sort(rng.choice(w.N, 256, replace=False)))]
    err = grad_errors(inp, {"dq": dq.cpu(), "dk": dk.cpu(), "dv": dv.cpu()}, w.scale, True, [(0, 3)], sampled)
    assert max(err.values()) <= GRAD_TOL, err


@pytest.mark.parametrize("B,H,Hkv,Nq,Nkv,d,window", [(3, 8, 2, 1, 2000, 128, -1), (2, 4, 4, 3, 700, 64, 50)])
def test_fp16_decode(B, H, Hkv, Nq, Nkv, d, window):
    inp = make_decode_inputs(B, H, Hkv, Nq, Nkv, d, seed=9600 + Nkv, lengths="mixed", tail_nan=True,
                             dtype=torch.float16)
    q, k, v, sl = (inp[n].cuda() for n in ("q", "k", "v", "seqlens"))
    o, lse = api.decode(q, k, v, sl, causal=True, window=None if window < 0 else window)
    torch.cuda.synchronize()
    assert api.get_status() == 0 and o.dtype == torch.float16
    eo, el = decode_errors(inp, o, lse, d ** -0.5, True, window)
    assert eo <= O_TOL and el <= LSE_TOL, (eo, el)


def test_mixed_dtypes_rejected():
    q = torch.zeros((1, 16, 2, 64), dtype=torch.float16, device="cuda")
    k = torch.zeros((1, 16, 2, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(TypeError):
        api.fwd(q, k, k)
