"""Backward parity: fa_bwd (CUDA, via the C ABI) against the fp64 oracle."""
import pytest
import torch

from exact_io_aware_93_b200 import api
from exact_io_aware_93_b200.inputs import (WORKLOADS, head_row_seed, make_inputs,
                                            make_workload_inputs, sample_rows)
from tests.parity import GRAD_TOL, grad_errors

pytestmark = pytest.mark.gpu


def _run(inp, causal, scale=None):
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = api.fwd(q, k, v, causal=causal, scale=scale)
    dq, dk, dv = api.bwd(q, k, v, o, do, lse, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert api.get_status() == 0
    return {"dq": dq.cpu(), "dk": dk.cpu(), "dv": dv.cpu()}


SMALL = [(1, 1, 1, 64), (1, 2, 7, 128), (2, 1, 129, 64), (1, 2, 256, 128), (1, 1, 300, 128),
         (2, 2, 500, 64), (1, 1, 640, 128)]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,H,N,d", SMALL)
def test_bwd_small_and_ragged(B, H, N, d, causal):
    inp = make_inputs(B, H, N, d, seed=8000 + N + d, with_do=True)
    g = _run(inp, causal)
    heads = [(b, h) for b in range(B) for h in range(H)]
    err = grad_errors(inp, g, d ** -0.5, causal, heads, [])
    assert max(err.values()) <= GRAD_TOL, err


def test_bwd_workload_fwdbwd_causal():
    w = WORKLOADS["causal_fwdbwd_b2_h16_n8192_d128"]
    inp = make_workload_inputs(w)
    g = _run(inp, w.causal)
    full = [(0, 0), (1, 15)]
    sampled = []
    for b, h in [(0, 5), (0, 11), (1, 2), (1, 9)][: w.bwd_extra_heads]:
        rows = sample_rows(w.N, w.bwd_extra_rows, head_row_seed(w.seed, b, h)).numpy()
        sampled.append((b, h, rows))
    err = grad_errors(inp, g, w.scale, w.causal, full, sampled)
    print("fwd+bwd workload gradient errors:", err)
    assert max(err.values()) <= GRAD_TOL, err


@pytest.mark.parametrize("B,H,N", [(2, 3, 12000), (1, 7, 10000)])
def test_bwd_grid_groups_with_a_ragged_last_group(B, H, N):
    """The backward grid walks (batch, head) pairs in groups sized to L2 (here 4 + 2 and
    5 + 2 heads): every head of every group, sampled rows, against the oracle."""
    d = 128
    inp = make_inputs(B, H, N, d, seed=8100 + N, with_do=True)
    g = _run(inp, True)
    sampled = [(b, h, sample_rows(N, 48, head_row_seed(8100 + N, b, h)).numpy())
               for b in range(B) for h in range(H)]
    err = grad_errors(inp, g, d ** -0.5, True, [], sampled)
    assert max(err.values()) <= GRAD_TOL, err


def test_bwd_nondefault_scale():
    inp = make_inputs(1, 2, 384, 128, seed=77, with_do=True)
    g = _run(inp, True, scale=0.21)
    err = grad_errors(inp, g, 0.21, True, [(0, 0), (0, 1)], [])
    assert max(err.values()) <= GRAD_TOL, err


def test_bwd_dk_dv_deterministic_and_dk_sums_to_zero():
    inp = make_inputs(1, 4, 2048, 128, seed=31, with_do=True)
    g1 = _run(inp, True)
    g2 = _run(inp, True)
    assert torch.equal(g1["dk"], g2["dk"]) and torch.equal(g1["dv"], g2["dv"])
    # sum over keys of dK_j = scale * sum_i q_i sum_j dS_ij = 0 (rows of dS sum to zero)
    s = g1["dk"].float().sum(dim=1)                     # [B, H, d]
    scale_ref = g1["dk"].float().abs().amax()
    assert float(s.abs().max()) <= 2e-2 * float(scale_ref) * 8, float(s.abs().max())


def test_bwd_workspace_checks():
    q = torch.zeros(1, 128, 1, 64, dtype=torch.bfloat16, device="cuda")
    o, lse = api.fwd(q, q, q)
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(api.FAError) as e:
        api.bwd(q, q, q, o, q, lse, workspace=small)
    assert e.value.status == 7
    assert api.bwd_workspace_size(2, 3, 100, 128) == 4 * 2 * 3 * (100 * 128 + 2 * 128)
