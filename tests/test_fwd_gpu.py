"""Forward parity: fa_fwd (CUDA, via the C ABI) against the fp64 oracle."""
import pytest
import torch

from exact_io_aware_93_b200 import api
from exact_io_aware_93_b200.inputs import WORKLOADS, make_inputs, make_workload_inputs
from tests.parity import LSE_TOL, O_TOL, fwd_errors

pytestmark = pytest.mark.gpu


def _run(inp, causal, scale=None):
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    o, lse = api.fwd(q, k, v, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert api.get_status() == 0
    return o, lse


SMALL = [(b, h, n, d) for (b, h, n) in [(1, 1, 1), (2, 3, 7), (1, 2, 127), (1, 1, 128), (2, 1, 129),
                                         (1, 2, 255), (1, 1, 256), (2, 2, 257), (1, 3, 384), (1, 2, 1000)]
         for d in (64, 128)]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,H,N,d", SMALL)
def test_fwd_small_and_ragged(B, H, N, d, causal):
    inp = make_inputs(B, H, N, d, seed=7000 + N + d)
    o, lse = _run(inp, causal)
    eo, el, where = fwd_errors(inp, o, lse, d ** -0.5, causal)
    assert eo <= O_TOL and el <= LSE_TOL, (eo, el, where)


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_fwd_workloads(name):
    w = WORKLOADS[name]
    inp = make_workload_inputs(w)
    o, lse = _run(inp, w.causal)
    eo, el, where = fwd_errors(inp, o, lse, w.scale, w.causal, w.rows_per_head, w.seed)
    print(f"{name}: max|dO|={eo:.3e} max rel dLSE={el:.3e} at {where}")
    assert eo <= O_TOL and el <= LSE_TOL, (eo, el, where)


def test_fwd_nondefault_scale_and_example_shape():
    # the flash_attn_func example call of the holysheep.ai review: B=4, N=16384, H=16, d=64, causal
    inp = make_inputs(4, 16, 16384, 64, seed=4242)
    o, lse = _run(inp, True, scale=0.3)
    eo, el, where = fwd_errors(inp, o, lse, 0.3, True, rows_per_head=64, seed=4242,
                               heads=[(0, 0), (3, 15), (1, 7)])
    assert eo <= O_TOL and el <= LSE_TOL, (eo, el, where)


def test_fwd_deterministic():
    inp = make_inputs(2, 4, 3000, 128, seed=99)
    o1, l1 = _run(inp, True)
    o2, l2 = _run(inp, True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_fwd_causal_future_blind():
    inp = make_inputs(1, 2, 700, 128, seed=5)
    o1, l1 = _run(inp, True)
    cut = 300
    inp2 = dict(inp)
    inp2["k"] = inp["k"].clone()
    inp2["v"] = inp["v"].clone()
    inp2["k"][:, cut + 1:] = -inp2["k"][:, cut + 1:] * 2
    inp2["v"][:, cut + 1:] = 7.0
    o2, l2 = _run(inp2, True)
    assert torch.equal(o1[:, : cut + 1], o2[:, : cut + 1])
    assert torch.equal(l1[:, :, : cut + 1], l2[:, :, : cut + 1])


def test_fwd_allocates_no_workspace():
    inp = make_inputs(1, 4, 4096, 128, seed=3)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    o = torch.empty_like(q)
    lse = torch.empty((1, 4, 4096), dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    torch.cuda.reset_peak_memory_stats()
    base = torch.cuda.memory_allocated()
    api.fwd(q, k, v, causal=True, out=o, lse=lse)
    torch.cuda.synchronize()
    assert torch.cuda.max_memory_allocated() == base


def test_fwd_rejects_bad_inputs():
    q = torch.zeros(1, 8, 2, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        api.fwd(q, q[:, :4], q[:, :4])
    with pytest.raises(api.FAError) as e:
        z = torch.zeros(1, 8, 2, 96, dtype=torch.bfloat16, device="cuda")
        api.fwd(z, z, z)
    assert e.value.status == 2
    with pytest.raises(TypeError):
        api.fwd(q.float(), q.float(), q.float())
