"""Seeded random configurations through the forward, backward and decode entry points,
against the fp64 oracle: batch, heads, grouping, lengths, head dimension, masking and
element type drawn together, so that combinations no hand-written case names get checked.
FA_FUZZ_DRAWS=n widens each draw to n seeds (default 24)."""
import os

import numpy as np
import pytest
import torch

from exact_io_aware_93_b200 import api
from exact_io_aware_93_b200.inputs import make_decode_inputs, make_inputs
from tests.parity import GRAD_TOL, LSE_TOL, O_TOL, decode_errors, fwd_errors, fwd_errors_gqa, grad_errors_gqa

pytestmark = pytest.mark.gpu
_DRAWS = int(os.environ.get("FA_FUZZ_DRAWS", "0"))


def _fwdbwd_case(seed):
    rng = np.random.default_rng(seed)
    h_kv = int(rng.choice([1, 2, 3]))
    H = h_kv * int(rng.choice([1, 2, 4]))
    N = int(rng.choice([1, 2, 63, 64, 65, 127, 129, 200, 255, 384, 511, 700]))
    d = int(rng.choice([64, 128]))
    causal = bool(rng.integers(0, 2))
    window = int(rng.choice([-1, -1, 0, 1, 17, 128, 300])) if causal else -1
    dtype = torch.float16 if rng.integers(0, 3) == 0 else torch.bfloat16
    return dict(B=int(rng.integers(1, 3)), H=H, H_kv=h_kv, N=N, d=d, causal=causal, window=window, dtype=dtype)


@pytest.mark.parametrize("seed", range(_DRAWS or 24))
def test_fuzz_fwd_bwd(seed):
    c = _fwdbwd_case(10_000 + seed)
    inp = make_inputs(c["B"], c["H"], c["N"], c["d"], seed=20_000 + seed, with_do=True, H_kv=c["H_kv"],
                      dtype=c["dtype"])
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "do"))
    w = None if c["window"] < 0 else c["window"]
    o, lse = api.fwd(q, k, v, causal=c["causal"], window=w)
    dq, dk, dv = api.bwd(q, k, v, o, do, lse, causal=c["causal"], window=w)
    torch.cuda.synchronize()
    assert api.get_status() == 0, c
    if c["H_kv"] == c["H"] and c["window"] < 0:
        # plain multi-head attention: the five configurations' gate, max |O - O_ref| itself
        eo, el, where = fwd_errors(inp, o, lse, c["d"] ** -0.5, c["causal"])
    else:
        # grouped heads or a window: rows may see one or two keys, where the output's own
        # rounding reaches 1e-2; judged by the excess over half an ulp (tests/parity.py)
        eo, el = fwd_errors_gqa(inp, o, lse, c["d"] ** -0.5, c["causal"], c["window"])
    assert eo <= O_TOL and el <= LSE_TOL, (c, eo, el)
    # gradients: the error in excess of the roundings the method performs by design (O in D,
    # P, dS, the outputs; tests/parity.py), which dominate near-zero gradients of rows that
    # see one or two keys
    err = grad_errors_gqa(inp, {"dq": dq.cpu(), "dk": dk.cpu(), "dv": dv.cpu()}, c["d"] ** -0.5, c["causal"],
                          c["window"], bounded=True)
    assert max(err.values()) <= GRAD_TOL, (c, err)


def _decode_case(seed):
    rng = np.random.default_rng(seed)
    h_kv = int(rng.choice([1, 2, 4]))
    G = int(rng.choice([1, 2, 4, 8, 16]))
    n_q = int(rng.choice([1, 1, 2, 3, 8]))
    while G * n_q > 128:
        n_q //= 2
    n_kv = int(rng.choice([1, 100, 128, 129, 1000, 3000]))
    B = int(rng.integers(1, 6))
    lens = [int(x) for x in rng.integers(0, n_kv + 1, B)]
    causal = bool(rng.integers(0, 4) > 0)
    window = int(rng.choice([-1, -1, 0, 5, 200])) if causal else -1
    dtype = torch.float16 if rng.integers(0, 3) == 0 else torch.bfloat16
    return dict(B=B, H=G * h_kv, H_kv=h_kv, N_q=n_q, N_kv=n_kv, d=int(rng.choice([64, 128])), lens=lens,
                causal=causal, window=window, dtype=dtype)


@pytest.mark.parametrize("seed", range(_DRAWS or 24))
def test_fuzz_decode(seed):
    c = _decode_case(30_000 + seed)
    inp = make_decode_inputs(c["B"], c["H"], c["H_kv"], c["N_q"], c["N_kv"], c["d"], seed=40_000 + seed,
                             lengths=c["lens"], tail_nan=True, dtype=c["dtype"])
    q, k, v, sl = (inp[n].cuda() for n in ("q", "k", "v", "seqlens"))
    o, lse = api.decode(q, k, v, sl, causal=c["causal"], window=None if c["window"] < 0 else c["window"])
    torch.cuda.synchronize()
    assert api.get_status() == 0, c
    eo, el = decode_errors(inp, o, lse, c["d"] ** -0.5, c["causal"], c["window"])
    assert eo <= O_TOL and el <= LSE_TOL, (c, eo, el)
