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


# nvidia-smi rows in the order of ClockSampler.QUERY
_ROW = "{ts}, 0, {sm} MHz, 1965 MHz, {pw} W, 0x0, Not Active, Not Active, Not Active, {cap}"


def _rows(specs):
    return [_ROW.format(ts=ts, sm=sm, pw=pw, cap="Active" if cap else "Not Active") for ts, sm, pw, cap in specs]


def test_clock_samples_parse_and_window():
    rows = _rows([("2026/12/02 10:00:00.000", 1965, 300, False),
                  ("2026/12/02 10:00:00.200", 1800, 900, True),
                  ("2026/12/02 10:00:01.000", 1500, 1000, True)])
    samples = bench.parse_clock_samples(rows + ["garbage", ""])
    assert len(samples) == 3
    assert samples[1]["reasons"] == ["sw_power_cap"] and samples[0]["reasons"] == []
    t0 = samples[0]["ts"]
    st = bench.clock_stats(samples, (t0, t0 + 0.3))
    assert st["samples"] == 2 and st["power_cap_samples"] == 1
    assert st["sm_mhz"] == (1965 + 1800) / 2 and st["sm_max_mhz"] == 1965 and st["power_w_max"] == 900
    assert st["reasons"] == ["sw_power_cap"]
    assert bench.clock_stats(samples, (t0 + 5, t0 + 6))["samples"] == 0


def test_peak_follows_the_regions_own_clock_samples():
    burst, sus = 1652.2, 1379.2
    # no in-region sample saw the power cap: burst peak, and the rule says on how many samples
    peak, kind, rule = bench.choose_peak({"samples": 3, "power_cap_samples": 0}, burst, sus)
    assert (peak, kind) == (burst, "burst") and "0 of 3" in rule
    # a capped sample or two in a mostly uncapped region: still the burst peak
    peak, kind, rule = bench.choose_peak({"samples": 5, "power_cap_samples": 1}, burst, sus)
    assert (peak, kind) == (burst, "burst") and "1 of 5" in rule
    peak, kind, _ = bench.choose_peak({"samples": 6, "power_cap_samples": 3}, burst, sus)
    assert (peak, kind) == (burst, "burst")
    # a capped majority: the sustained peak
    peak, kind, rule = bench.choose_peak({"samples": 24, "power_cap_samples": 15}, burst, sus)
    assert (peak, kind) == (sus, "sustained") and "15 of 24" in rule
    # no samples at all: the burst peak (the larger denominator, so the smaller fraction)
    peak, kind, _ = bench.choose_peak({"samples": 0, "power_cap_samples": 0}, burst, sus)
    assert peak == burst


def test_per_config_covers_the_metrics_range():
    from exact_io_aware_93_b200.inputs import WORKLOADS
    ns = sorted(WORKLOADS[n].N for n in bench.PER_CONFIG)
    assert ns == [2048, 8192, 32768, 131072]
    assert all(WORKLOADS[n].causal for n in bench.PER_CONFIG)
    assert bench.DEFAULT_WORKLOAD in bench.PER_CONFIG
