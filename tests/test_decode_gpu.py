"""Decoding (few new queries per sequence against a key/value cache) through fa_decode,
against the fp64 oracle."""
import numpy as np
import pytest
import torch

from exact_io_aware_93_b200 import api
from exact_io_aware_93_b200.inputs import DECODE_WORKLOADS, make_decode_inputs, make_decode_workload_inputs
from tests.parity import LSE_TOL, O_TOL, decode_errors

pytestmark = pytest.mark.gpu

CASES = [
    # B, H, H_kv, N_q, N_kv, d, causal, window, lengths, stale tail = NaN
    (1, 1, 1, 1, 1, 64, True, -1, "full", False),                  # one key
    (3, 8, 2, 1, 1000, 128, True, -1, [1000, 1, 517], True),       # ragged lengths, 4 heads per group
    (2, 32, 8, 1, 2000, 128, True, -1, "mixed", True),             # the 8B head layout
    (2, 4, 4, 3, 700, 64, True, -1, [700, 2], False),              # N_q > a cached length
    (2, 8, 1, 4, 900, 128, False, -1, [900, 300], True),           # multi-query, non-causal
    (2, 16, 2, 8, 1300, 128, True, 100, [1300, 129], True),        # window, 64 rows per tile
    (1, 128, 1, 1, 5000, 128, True, -1, "full", False),            # 128 rows: a full tile
    (4, 8, 8, 1, 257, 64, True, 0, "mixed", False),                # window 0: the key at the query
    (2, 4, 2, 2, 3000, 128, True, -1, [0, 3000], True),            # an empty cache
    (64, 8, 8, 1, 300, 128, True, -1, "mixed", True),              # many pairs per CTA
    (2, 8, 2, 16, 700, 64, True, 255, [700, 650], False),          # verifying 16 drafted tokens
]


@pytest.mark.parametrize("B,H,Hkv,Nq,Nkv,d,causal,window,lengths,tail_nan", CASES)
def test_decode_parity(B, H, Hkv, Nq, Nkv, d, causal, window, lengths, tail_nan):
    inp = make_decode_inputs(B, H, Hkv, Nq, Nkv, d, seed=9300 + Nkv + H + Nq, lengths=lengths, tail_nan=tail_nan)
    q, k, v, sl = (inp[n].cuda() for n in ("q", "k", "v", "seqlens"))
    w = None if window < 0 else window
    o, lse = api.decode(q, k, v, sl, causal=causal, window=w)
    torch.cuda.synchronize()
    assert api.get_status() == 0
    eo, el = decode_errors(inp, o, lse, d ** -0.5, causal, window)
    assert eo <= O_TOL and el <= LSE_TOL, (eo, el)


def test_decode_split_across_ctas_and_full_caches():
    """One long sequence per head: every pair is split over many CTAs and merged; and
    seqlens = None reads every cache as full."""
    inp = make_decode_inputs(1, 4, 1, 1, 40000, 128, seed=9401, lengths="full")
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    o, lse = api.decode(q, k, v, None, causal=True)
    o2, lse2 = api.decode(q, k, v, inp["seqlens"].cuda(), causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(lse, lse2)
    eo, el = decode_errors(inp, o, lse, 128 ** -0.5, True)
    assert eo <= O_TOL and el <= LSE_TOL, (eo, el)


def test_decode_deterministic():
    inp = make_decode_inputs(3, 8, 2, 2, 5000, 128, seed=9402, lengths="mixed")
    q, k, v, sl = (inp[n].cuda() for n in ("q", "k", "v", "seqlens"))
    o1, l1 = api.decode(q, k, v, sl)
    o2, l2 = api.decode(q, k, v, sl)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_decode_graph_replay_reads_new_lengths():
    """The lengths are read by the kernels: a captured graph replayed after the lengths
    grow gives the new result."""
    inp = make_decode_inputs(4, 8, 2, 1, 3000, 128, seed=9403, lengths=[1000, 2000, 10, 2999])
    q, k, v, sl = (inp[n].cuda() for n in ("q", "k", "v", "seqlens"))
    out = torch.empty_like(q)
    lse = torch.empty((4, 8, 1), dtype=torch.float32, device="cuda")
    ws = torch.empty(api.decode_workspace_size(q, k), dtype=torch.uint8, device="cuda")
    api.decode(q, k, v, sl, out=out, lse=lse, workspace=ws)   # first call outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        api.decode(q, k, v, sl, out=out, lse=lse, workspace=ws)
    new_lens = torch.tensor([1001, 2500, 11, 3000], dtype=torch.int32)
    sl.copy_(new_lens)
    g.replay()
    torch.cuda.synchronize()
    inp["seqlens"] = new_lens
    eo, el = decode_errors(inp, out, lse, 128 ** -0.5, True)
    assert eo <= O_TOL and el <= LSE_TOL, (eo, el)
    del g


def test_decode_argument_errors():
    q = torch.zeros((2, 1, 8, 128), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((2, 64, 2, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(api.FAError):
        api.decode(q, k, k, None, causal=False, window=3)          # window without causal
    big = torch.zeros((2, 17, 8, 128), dtype=torch.bfloat16, device="cuda")
    kk = torch.zeros((2, 64, 1, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(api.FAError):
        api.decode(big, kk, kk)                                    # 8 x 17 rows > 128
    with pytest.raises(ValueError):
        api.decode(q, k, k, torch.zeros(2, dtype=torch.int64, device="cuda"))
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(api.FAError):
        api.decode(q, k, k, workspace=ws)                          # too small


@pytest.mark.parametrize("name", sorted(DECODE_WORKLOADS))
def test_decode_workload_sampled(name):
    """The full-size decode workload, in the launch configuration the benchmark times,
    checked on a seeded sample of (sequence, head) pairs."""
    w = DECODE_WORKLOADS[name]
    inp = make_decode_workload_inputs(w)
    q, k, v, sl = (inp[n].cuda() for n in ("q", "k", "v", "seqlens"))
    o, lse = api.decode(q, k, v, sl, causal=w.causal, window=None if w.window < 0 else w.window)
    torch.cuda.synchronize()
    assert api.get_status() == 0
    rng = np.random.default_rng(w.seed)
    pairs = sorted({(int(rng.integers(w.B)), int(rng.integers(w.H))) for _ in range(w.checked_heads)})
    pairs += [(0, 0), (w.B - 1, w.H - 1)]
    eo, el = decode_errors(inp, o, lse, w.scale, w.causal, w.window, heads=pairs)
    assert eo <= O_TOL and el <= LSE_TOL, (eo, el)
