"""The seeded workload generator (CPU)."""
import torch

from exact_io_aware_93_b200.inputs import WORKLOADS, make_inputs, sample_rows


def test_deterministic_and_bf16():
    a = make_inputs(2, 3, 17, 8, 42, with_do=True)
    b = make_inputs(2, 3, 17, 8, 42, with_do=True)
    for n in ("q", "k", "v", "do"):
        assert a[n].dtype == torch.bfloat16 and a[n].shape == (2, 17, 3, 8)
        assert torch.equal(a[n], b[n])
    c = make_inputs(2, 3, 17, 8, 43)
    assert not torch.equal(a["q"], c["q"])
    d = make_inputs(2, 3, 17, 8, 42)
    for n in ("q", "k", "v"):
        assert torch.equal(a[n], d[n])


def test_peaked_positions_scaled():
    plain = make_inputs(1, 2, 1000, 16, 7)
    peak = make_inputs(1, 2, 1000, 16, 7, peaked=True)
    pos = peak["peaked_positions"]
    assert pos.numel() == 10 and torch.unique(pos).numel() == 10
    mask = torch.zeros(1000, dtype=torch.bool)
    mask[pos] = True
    assert torch.equal(peak["k"][:, ~mask], plain["k"][:, ~mask])
    ratio = peak["k"][:, mask].float().abs().mean() / plain["k"][:, mask].float().abs().mean()
    assert 2.9 < ratio < 3.1
    assert torch.equal(peak["q"], plain["q"]) and torch.equal(peak["v"], plain["v"])


def test_sample_rows():
    r = sample_rows(32768, 4096, 5)
    assert r.numel() >= 4096 and r.numel() <= 4099
    assert torch.all(r[1:] > r[:-1])
    assert {0, 1, 32767} <= set(r.tolist())
    assert torch.equal(sample_rows(300, None, 1), torch.arange(300))
    assert torch.equal(r, sample_rows(32768, 4096, 5))


def test_workloads_table():
    assert len(WORKLOADS) == 5
    w = WORKLOADS["causal_fwdbwd_b2_h16_n8192_d128"]
    assert (w.B, w.H, w.N, w.d, w.causal, w.backward) == (2, 16, 8192, 128, True, True)
    assert abs(w.scale - 128 ** -0.5) < 1e-15


def test_decode_inputs_recipe():
    from exact_io_aware_93_b200.inputs import DECODE_WORKLOADS, make_decode_inputs
    a = make_decode_inputs(3, 4, 2, 2, 300, 64, 5, lengths="mixed")
    b = make_decode_inputs(3, 4, 2, 2, 300, 64, 5, lengths="mixed")
    assert a["q"].shape == (3, 2, 4, 64) and a["k"].shape == (3, 300, 2, 64)
    for n in ("q", "k", "v", "seqlens"):
        assert torch.equal(a[n], b[n])
    assert a["seqlens"].dtype == torch.int32
    assert torch.all((a["seqlens"] >= 150) & (a["seqlens"] <= 300))
    full = make_decode_inputs(3, 4, 2, 2, 300, 64, 5, lengths="full")
    assert torch.equal(full["q"], a["q"]) and torch.all(full["seqlens"] == 300)
    t = make_decode_inputs(2, 2, 1, 1, 10, 8, 6, lengths=[4, 10], tail_nan=True)
    assert torch.isnan(t["k"][0, 4:]).all() and not torch.isnan(t["k"][0, :4]).any()
    assert not torch.isnan(t["v"][1]).any()
    w = next(iter(DECODE_WORKLOADS.values()))
    assert w.N_kv % 128 == 0 and w.H % w.H_kv == 0
