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
