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
