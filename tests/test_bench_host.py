"""Host-side logic of bench.py: the FLOP and byte conventions its JSON line reports, and the
rule that ncu traffic figures count only for the kernel sources they were taken from."""
import json

import pytest

import bench

# (B, H, N, d, causal) of the five configurations and the forward FLOPs of the convention:
# 4 B H N^2 d, halved when causal
CONFIGS = [
    ((1, 1, 256, 64, False), 1.68e7),
    ((4, 16, 2048, 128, True), 6.87e10),
    ((1, 32, 32768, 128, True), 8.80e12),
    ((2, 16, 8192, 128, True), 5.50e11),
    ((1, 8, 131072, 128, True), 3.52e13),
]


@pytest.mark.parametrize("cfg,expected", CONFIGS)
def test_forward_flop_convention(cfg, expected):
    B, H, N, d, causal = cfg
    f = bench.fwd_flops(B, H, N, d, causal)
    assert f == 4.0 * B * H * N * N * d / (2 if causal else 1)
    assert abs(f - expected) / expected < 5e-3
    assert bench.bwd_flops(B, H, N, d, causal) == 2.5 * f


def test_window_counts_fewer_pairs_than_causal():
    full = bench.fwd_flops(1, 32, 32768, 128, True)
    win = bench.fwd_flops(1, 32, 32768, 128, True, 4096)
    assert win < full
    # every query sees at most window + 1 keys
    assert win <= 4.0 * 32 * 128 * 32768 * 4097


def test_forward_algorithmic_bytes():
    # Q, K, V read and O written in bf16, LSE written in fp32
    assert bench.fwd_bytes(2, 16, 8192, 128) == 2 * 4 * 2 * 16 * 8192 * 128 + 4 * 2 * 16 * 8192


def test_traffic_only_for_matching_sources(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "traffic.json").write_text(json.dumps(
        {"fa_bwd": {"w": {"dram_bytes_per_launch": 123, "source_digest": "abc"}}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_digest", lambda: "abc")
    assert bench.measured_traffic("fa_bwd", "w") == 123
    assert bench.measured_traffic("fa_bwd", "other") is None
    assert bench.measured_traffic("fa_fwd_kernel", "w") is None
    monkeypatch.setattr(bench, "kernel_source_digest", lambda: "changed")
    assert bench.measured_traffic("fa_bwd", "w") is None


def test_source_digest_is_stable():
    assert bench.kernel_source_digest() == bench.kernel_source_digest()
    assert len(bench.kernel_source_digest()) == 16
