"""Grouped-query / multi-query attention and causal sliding windows through fa_fwd_ex and
fa_bwd_ex, against the fp64 oracle."""
import pytest
import torch

from exact_io_aware_93_b200 import api
from exact_io_aware_93_b200.inputs import make_inputs
from tests.parity import GRAD_TOL, LSE_TOL, O_TOL, fwd_errors_gqa, grad_errors_gqa

pytestmark = pytest.mark.gpu

CASES = [
    # B, H, H_kv, N, d, causal, window
    (2, 8, 2, 300, 128, True, -1),      # grouped query
    (1, 4, 1, 1000, 64, False, -1),     # multi query, non-causal
    (1, 3, 1, 257, 128, True, -1),      # multi query, ragged
    (1, 2, 2, 1000, 128, True, 0),      # window 0: each query sees only itself
    (1, 2, 2, 1000, 128, True, 1),
    (1, 2, 2, 1000, 128, True, 127),
    (1, 2, 2, 1000, 128, True, 128),
    (2, 2, 2, 777, 64, True, 300),
    (1, 2, 2, 600, 128, True, 5000),    # window wider than the sequence = plain causal
    (1, 6, 3, 700, 128, True, 200),     # grouped query + window
]


@pytest.mark.parametrize("B,H,Hkv,N,d,causal,window", CASES)
def test_fwd_bwd_gqa_window(B, H, Hkv, N, d, causal, window):
    inp = make_inputs(B, H, N, d, seed=9100 + N + H + window, with_do=True, H_kv=Hkv)
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "do"))
    w = None if window < 0 else window
    o, lse = api.fwd(q, k, v, causal=causal, window=w)
    dq, dk, dv = api.bwd(q, k, v, o, do, lse, causal=causal, window=w)
    torch.cuda.synchronize()
    assert api.get_status() == 0
    eo, el = fwd_errors_gqa(inp, o, lse, d ** -0.5, causal, window)
    assert eo <= O_TOL and el <= LSE_TOL, (eo, el)
    err = grad_errors_gqa(inp, {"dq": dq.cpu(), "dk": dk.cpu(), "dv": dv.cpu()}, d ** -0.5, causal, window)
    assert max(err.values()) <= GRAD_TOL, err
    assert dk.shape == k.shape and dv.shape == v.shape


def test_window_equals_causal_when_wide():
    inp = make_inputs(1, 2, 900, 128, seed=77)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    o1, l1 = api.fwd(q, k, v, causal=True)
    o2, l2 = api.fwd(q, k, v, causal=True, window=899)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_ex_argument_checks():
    q = torch.zeros(1, 64, 4, 64, dtype=torch.bfloat16, device="cuda")
    k3 = torch.zeros(1, 64, 3, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        api.fwd(q, k3, k3)                      # 3 key/value heads do not divide 4 query heads
    with pytest.raises(api.FAError) as e:
        api.fwd(q, q, q, causal=False, window=8)  # a window needs causal masking
    assert e.value.status == 1
