"""The parity helpers' own arithmetic (CPU)."""
import numpy as np
import torch

from exact_io_aware_93_b200.accounting import visible_pairs
from tests.parity import bf16_half_ulp


def test_bf16_half_ulp_matches_torch_rounding():
    for x in (1.0, 1.5, 2.0, 3.875, 4.0, -5.0, 0.296875, 100.0, 1e-3):
        xb = float(torch.tensor(x).to(torch.bfloat16))
        h = float(bf16_half_ulp(np.array([xb]))[0])
        assert float(torch.tensor(xb + 0.99 * h, dtype=torch.float64).to(torch.bfloat16)) == xb
        assert float(torch.tensor(xb + 1.01 * h, dtype=torch.float64).to(torch.bfloat16)) != xb


def test_visible_pairs_counts():
    for n, w in [(10, 3), (100, 0), (100, 99), (1000, 128), (7, 50)]:
        brute = sum(min(i, w) + 1 for i in range(n))
        assert visible_pairs(n, True, w) == brute
    assert visible_pairs(8192, True) == 8192 * 8192 / 2
    assert visible_pairs(100, False) == 100 * 100


def test_half_ulp_fp16_matches_torch_rounding():
    from tests.parity import half_ulp
    for x in (1.0, 1.5, 3.0, -7.25, 0.1, 300.0):
        xh = float(torch.tensor(x).to(torch.float16))
        h = float(half_ulp(np.array([xh]), torch.float16)[0])
        assert float(torch.tensor(xh + 0.99 * h, dtype=torch.float64).to(torch.float16)) == xh
        assert float(torch.tensor(xh + 1.01 * h, dtype=torch.float64).to(torch.float16)) != xh


def test_decode_accounting_brute_force():
    """Bytes and FLOPs the decode benchmark reports, against a brute-force count of the
    visible (query, key) pairs and cache rows."""
    from exact_io_aware_93_b200.accounting import decode_bytes, decode_cache_keys, decode_flops
    lens, H, H_kv, n_q, d = [0, 5, 37, 200], 8, 2, 3, 16
    for causal, window in ((True, -1), (False, -1), (True, 0), (True, 10)):
        pairs, rows = 0, 0
        for n in lens:
            seen = set()
            for i in range(n_q):
                pos = n - n_q + i if causal else n - 1
                for j in range(n):
                    vis = (j <= pos and (window < 0 or j >= pos - window)) if causal else True
                    if pos >= 0 and vis:
                        pairs += 1
                        seen.add(j)
            rows += len(seen)
            assert decode_cache_keys(n, n_q, causal, window) >= len(seen)
        assert decode_flops(lens, H, n_q, d, causal, window) == 4.0 * d * H * pairs
        if window < 0 or not causal:
            assert decode_bytes(lens, 4, H, H_kv, n_q, d, causal, window) == \
                4 * d * H_kv * rows + 4 * 4 * n_q * H * d + 4 * 4 * H * n_q + 4 * 4


def test_e4m3_quantisation_recipe():
    from exact_io_aware_93_b200.inputs import make_inputs_e4m3, quantize_e4m3
    x = torch.tensor([0.0, 1.0, -3.0, 448.0 / 3.0])
    codes, ds = quantize_e4m3(x)
    assert codes.dtype == torch.float8_e4m3fn
    assert abs(codes.float().abs().max().item() - 448.0) < 1e-6          # amax maps to the top code
    assert np.allclose(codes.float().numpy() * ds, x.numpy(), rtol=2 ** -4)
    t = make_inputs_e4m3(1, 2, 40, 128, seed=3, H_kv=1)
    assert t["q"].shape == (1, 40, 2, 128) and t["k"].shape == (1, 40, 1, 128)
    assert all(isinstance(t[n + "_descale"], float) and t[n + "_descale"] > 0 for n in "qkv")


def _rounded_backward(q, k, v, do, scale, causal, window, dtype, drop_d=False):
    """fp64 backward with exactly the roundings grad_rounding_bounds covers: O and P rounded to
    `dtype`, D from the rounded O, dS rounded to `dtype`.  drop_d plants a real mistake."""
    import oracle
    o, _, p = oracle.dense_fwd(q, k, v, scale, causal, window)

    def rnd(x):
        return torch.tensor(x).to(dtype).double().numpy()
    pt, ot = rnd(p), rnd(o)
    dp = do @ v.T
    dd = 0.0 if drop_d else (do * ot).sum(1)[:, None]
    ds = rnd(pt * (dp - dd))
    return scale * ds @ k, scale * ds.T @ q, pt.T @ do


def _small_problems():
    from exact_io_aware_93_b200.inputs import make_inputs
    rng = np.random.default_rng(5)
    for trial in range(40):
        n = int(rng.choice([1, 2, 3, 5, 17, 64, 130]))
        d = int(rng.choice([64, 128]))
        causal = bool(rng.integers(0, 2))
        window = int(rng.choice([-1, 0, 1, 9])) if causal else -1
        dtype = torch.float16 if trial % 3 == 0 else torch.bfloat16
        inp = make_inputs(1, 1, n, d, seed=700 + trial, with_do=True, dtype=dtype)
        head = [inp[x][0, :, 0, :].double().numpy() for x in ("q", "k", "v", "do")]
        yield head, d ** -0.5, causal, window, dtype


def test_grad_rounding_bound_contains_the_methods_roundings():
    """The bound holds element by element for a backward that performs exactly those
    roundings, on small problems including rows that see one or two keys."""
    import oracle
    from tests.parity import grad_rounding_bounds
    for (q, k, v, do), scale, causal, window, dtype in _small_problems():
        ref = oracle.bwd_rows(q, k, v, do, scale, causal, window=window)
        ref = (ref[0], ref[2], ref[3])
        got = _rounded_backward(q, k, v, do, scale, causal, window, dtype)
        bounds = grad_rounding_bounds(q, k, v, do, scale, causal, window, dtype)
        for g, r, bd in zip(got, ref, bounds):
            assert (np.abs(g - r) <= bd * (1 + 1e-9) + 1e-15).all()


def test_grad_rounding_bound_does_not_excuse_a_dropped_term():
    """Leaving D out of dS is caught: its error exceeds the bound by more than the tolerance."""
    import oracle
    from tests.parity import GRAD_TOL, grad_rounding_bounds
    caught = 0
    total = 0
    for (q, k, v, do), scale, causal, window, dtype in _small_problems():
        if q.shape[0] < 17:
            continue
        total += 1
        dq_ref = oracle.bwd_rows(q, k, v, do, scale, causal, window=window)[0]
        dq_bad = _rounded_backward(q, k, v, do, scale, causal, window, dtype, drop_d=True)[0]
        bq = grad_rounding_bounds(q, k, v, do, scale, causal, window, dtype)[0]
        excess = np.maximum(np.abs(dq_bad - dq_ref) - bq, 0.0).max() / max(np.abs(dq_ref).max(), 1e-3)
        caught += excess > GRAD_TOL
    assert total > 0 and caught == total
