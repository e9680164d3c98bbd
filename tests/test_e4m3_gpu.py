"""fp8 e4m3 forward through fa_fwd_e4m3_scaled, against the fp64 oracle on the dequantised
inputs, with the output bound that e4m3 rounding of the softmax weights allows."""
import pytest
import torch

from exact_io_aware_93_b200 import api
from exact_io_aware_93_b200.inputs import EXTRA_WORKLOADS, make_inputs_e4m3, make_workload_inputs
from tests.parity import LSE_TOL, fwd_errors_e4m3

pytestmark = pytest.mark.gpu

CASES = [
    # B, H, H_kv, N, causal, window
    (1, 2, 2, 1, False, -1),
    (1, 2, 2, 129, True, -1),
    (2, 4, 2, 300, False, -1),
    (1, 2, 1, 1000, True, -1),
    (1, 2, 2, 700, True, 100),
    (1, 4, 4, 257, True, 0),
]


@pytest.mark.parametrize("B,H,Hkv,N,causal,window", CASES)
def test_e4m3_forward(B, H, Hkv, N, causal, window):
    inp = make_inputs_e4m3(B, H, N, 128, seed=9700 + N + H, H_kv=Hkv)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    o, lse = api.fwd_e4m3(q, k, v, inp["q_descale"], inp["k_descale"], inp["v_descale"], causal=causal,
                          window=None if window < 0 else window)
    torch.cuda.synchronize()
    assert api.get_status() == 0 and o.dtype == torch.bfloat16
    excess, worst, el = fwd_errors_e4m3(inp, o, lse, 128 ** -0.5, causal, window)
    assert excess <= 0 and el <= LSE_TOL, (excess, worst, el)


def test_e4m3_workload_sampled():
    w = EXTRA_WORKLOADS["e4m3_causal_fwd_b2_h16_n8192_d128"]
    inp = make_workload_inputs(w)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    o, lse = api.fwd_e4m3(q, k, v, inp["q_descale"], inp["k_descale"], inp["v_descale"], causal=True)
    torch.cuda.synchronize()
    assert api.get_status() == 0
    excess, worst, el = fwd_errors_e4m3(inp, o, lse, w.scale, True, rows_per_head=w.rows_per_head, seed=w.seed,
                                        heads=[(0, 0), (1, 15), (0, 9)])
    assert excess <= 0 and el <= LSE_TOL, (excess, worst, el)


def test_e4m3_unit_descales_match_fwd_ex():
    inp = make_inputs_e4m3(1, 2, 500, 128, seed=9801)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    o1, l1 = api.fwd_e4m3(q, k, v, 1.0, 1.0, 1.0, causal=True, scale=0.01)
    o2, l2 = api.fwd(q, k, v, causal=True, scale=0.01)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_e4m3_rejections():
    q = torch.zeros((1, 16, 2, 64), dtype=torch.float8_e4m3fn, device="cuda")
    with pytest.raises(api.FAError):
        api.fwd_e4m3(q, q, q, 1.0, 1.0, 1.0)                        # d = 64 is not built for e4m3
    q = torch.zeros((1, 16, 2, 128), dtype=torch.float8_e4m3fn, device="cuda")
    with pytest.raises(api.FAError):
        api.fwd_e4m3(q, q, q, 0.0, 1.0, 1.0)                        # descale must be positive
    o, lse = api.fwd_e4m3(q, q, q, 1.0, 1.0, 1.0)
    do = torch.zeros((1, 16, 2, 128), dtype=torch.float8_e4m3fn, device="cuda")
    with pytest.raises(Exception):
        api.bwd(q, q, q, do, do, lse)                               # the e4m3 path is forward only
