"""Seeded synthetic workloads shared by the tests, the benchmark and the smoke check.

This module only draws random numbers and picks rows; it holds none of the
attention arithmetic, and neither the CUDA path nor the oracle depends on it.

Recipe (the same for every workload):

* ``torch.Generator('cpu')`` seeded with the workload's seed draws fp32
  standard normals in the order Q, K, V, dO, each of shape
  ``[B, N, H, d]`` (batch, sequence, heads, head_dim -- the layout of the
  ``flash_attn_func`` interface in the holysheep.ai review, section
  "Implementing Flash Attention in Your Architecture").
* For the peaked workload, a seeded permutation picks floor(N/100) sequence
  positions (shared by all batches and heads) and the whole K vector at those
  positions is multiplied by 3 in fp32, before rounding.
* Every tensor is then rounded to bfloat16 (round to nearest even), or to
  float16 where a test asks for fp16; the same 16-bit values are handed to the
  GPU and, widened exactly to fp64, to the oracle.
* Checked query rows: per (b, h) a seeded sample without replacement from
  [0, N), always including rows 0, 1 and N-1.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool
    seed: int
    backward: bool = False
    peaked: bool = False
    H_kv: int | None = None          # key/value heads (None: same as H)
    window: int = -1                 # causal sliding window (-1: none)
    dtype: str = "bf16"              # element type of the inputs: "bf16", "f16" or "e4m3" (forward only)
    # forward rows checked per head (None = every row)
    rows_per_head: int | None = None
    # backward: heads checked in full, plus (extra_heads x extra_rows_per_head) sampled rows
    bwd_full_heads: int = 0
    bwd_extra_heads: int = 0
    bwd_extra_rows: int = 0
    notes: str = field(default="", compare=False)

    @property
    def scale(self) -> float:
        return 1.0 / float(self.d) ** 0.5

    @property
    def torch_dtype(self) -> torch.dtype:
        return {"f16": torch.float16, "e4m3": torch.float8_e4m3fn}.get(self.dtype, torch.bfloat16)


# The five workloads: shapes, seeds and checked-row counts.
WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny_b1_h1_n256_d64", 1, 1, 256, 64, False, 1001,
                 notes="tiny non-causal forward, every row checked"),
        Workload("causal_b4_h16_n2048_d128", 4, 16, 2048, 128, True, 1002,
                 rows_per_head=None,
                 notes="causal forward, every row of every head checked"),
        Workload("causal_b1_h32_n32768_d128", 1, 32, 32768, 128, True, 1003,
                 rows_per_head=4096,
                 notes="long-context causal forward, 4096 rows per head"),
        Workload("causal_fwdbwd_b2_h16_n8192_d128", 2, 16, 8192, 128, True, 1004,
                 backward=True, bwd_full_heads=2, bwd_extra_heads=4, bwd_extra_rows=256,
                 notes="causal forward + recompute backward; 2 full heads + 1024 rows elsewhere"),
        Workload("causal_peaked_b1_h8_n131072_d128", 1, 8, 131072, 128, True, 1005,
                 peaked=True, rows_per_head=512,
                 notes="very long causal forward, K x3 on 1% of positions, 512 rows per head"),
    ]
}


# Workloads of the rows beyond the five configurations: grouped-query heads and a causal
# sliding window, at the shapes of common long-context models.
EXTRA_WORKLOADS = {
    w.name: w
    for w in [
        Workload("gqa_causal_fwdbwd_b2_h32_hkv8_n8192_d128", 2, 32, 8192, 128, True, 1101,
                 backward=True, H_kv=8,
                 notes="4 query heads per key/value head, causal forward + backward"),
        Workload("window4096_causal_fwdbwd_b1_h32_hkv8_n32768_d128", 1, 32, 32768, 128, True, 1102,
                 backward=True, H_kv=8, window=4096,
                 notes="grouped heads + causal sliding window of 4096 keys, forward + backward"),
        Workload("f16_causal_fwdbwd_b2_h16_n8192_d128", 2, 16, 8192, 128, True, 1104,
                 backward=True, dtype="f16", bwd_full_heads=1, bwd_extra_heads=2, bwd_extra_rows=256,
                 notes="the forward + backward configuration with fp16 tensors"),
        Workload("e4m3_causal_fwd_b2_h16_n8192_d128", 2, 16, 8192, 128, True, 1105,
                 dtype="e4m3", rows_per_head=256,
                 notes="fp8 e4m3 forward at the forward + backward configuration's shape"),
    ]
}


@dataclass(frozen=True)
class DecodeWorkload:
    """Decoding: N_q new queries per sequence against a key/value cache of capacity N_kv."""
    name: str
    B: int
    H: int
    H_kv: int
    N_q: int
    N_kv: int
    d: int
    causal: bool
    seed: int
    lengths: str = "mixed"           # "full": every sequence N_kv long; "mixed": see make_decode_inputs
    window: int = -1
    checked_heads: int = 8           # (b, h) pairs checked against the oracle at full size
    notes: str = field(default="", compare=False)

    @property
    def scale(self) -> float:
        return 1.0 / float(self.d) ** 0.5


# Decoding at the head counts of an 8B-class model with grouped key/value heads: one new
# token per sequence, 16 sequences whose cached lengths are spread over [N_kv / 2, N_kv].
DECODE_WORKLOADS = {
    w.name: w
    for w in [
        DecodeWorkload("decode_b16_h32_hkv8_nq1_nkv32768_d128", 16, 32, 8, 1, 32768, 128, True, 1201,
                       notes="one new token per sequence, cache lengths spread over [16384, 32768]"),
    ]
}


def make_decode_inputs(B: int, H: int, H_kv: int, N_q: int, N_kv: int, d: int, seed: int, *,
                       lengths="mixed", tail_nan: bool = False,
                       dtype: torch.dtype = torch.bfloat16) -> dict[str, torch.Tensor]:
    """CPU tensors for decoding: ``q`` [B, N_q, H, d], ``k``/``v`` [B, N_kv, H_kv, d] (the
    cache), bf16 unless ``dtype`` says float16, and ``seqlens`` int32 [B].

    Recipe: a ``torch.Generator('cpu')`` seeded with ``seed`` draws fp32 standard normals
    for q, k, v in that order, rounded to bf16; then the lengths: ``"full"`` gives N_kv
    for every sequence, ``"mixed"`` draws each uniformly from [N_kv // 2, N_kv] with the
    same generator, and a sequence of ints is taken as given.  With ``tail_nan`` the cache
    positions past each length are overwritten with NaN (stale cache slots must not matter).
    """
    gen = torch.Generator(device="cpu")
    gen.manual_seed(int(seed))
    out = {
        "q": torch.randn((B, N_q, H, d), generator=gen, dtype=torch.float32).to(dtype),
        "k": torch.randn((B, N_kv, H_kv, d), generator=gen, dtype=torch.float32).to(dtype),
        "v": torch.randn((B, N_kv, H_kv, d), generator=gen, dtype=torch.float32).to(dtype),
    }
    if isinstance(lengths, str):
        if lengths == "full":
            lens = torch.full((B,), N_kv, dtype=torch.int32)
        elif lengths == "mixed":
            lens = torch.randint(N_kv // 2, N_kv + 1, (B,), generator=gen, dtype=torch.int64).to(torch.int32)
        else:
            raise ValueError(f"unknown length recipe {lengths!r}")
    else:
        lens = torch.tensor([int(x) for x in lengths], dtype=torch.int32)
        if lens.numel() != B:
            raise ValueError("one length per sequence expected")
    out["seqlens"] = lens
    if tail_nan:
        for b in range(B):
            n = max(0, min(int(lens[b]), N_kv))
            out["k"][b, n:] = float("nan")
            out["v"][b, n:] = float("nan")
    return out


def make_decode_workload_inputs(w: DecodeWorkload) -> dict[str, torch.Tensor]:
    return make_decode_inputs(w.B, w.H, w.H_kv, w.N_q, w.N_kv, w.d, w.seed, lengths=w.lengths)


def peaked_positions(N: int, gen: torch.Generator) -> torch.Tensor:
    """floor(N/100) distinct sequence positions, drawn by a seeded permutation."""
    return torch.randperm(N, generator=gen)[: N // 100]


def make_inputs(B: int, H: int, N: int, d: int, seed: int, *, with_do: bool = False,
                peaked: bool = False, H_kv: int | None = None,
                dtype: torch.dtype = torch.bfloat16) -> dict[str, torch.Tensor]:
    """CPU tensors ``q`` (and ``do``) of shape [B, N, H, d] and ``k, v`` of shape
    [B, N, H_kv, d] (H_kv defaults to H), bf16 unless ``dtype`` says float16."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(int(seed))
    hkv = H if H_kv is None else int(H_kv)
    out = {}
    names = ["q", "k", "v"] + (["do"] if with_do else [])
    for name in names:
        heads = hkv if name in ("k", "v") else H
        out[name] = torch.randn((B, N, heads, d), generator=gen, dtype=torch.float32)
    if peaked:
        pos = peaked_positions(N, gen)
        out["k"][:, pos] *= 3.0
        out["peaked_positions"] = pos
    for name in names:
        out[name] = out[name].to(dtype)
    return out


def quantize_e4m3(x: torch.Tensor) -> tuple[torch.Tensor, float]:
    """Per-tensor e4m3 quantisation: descale = fp32(amax / 448), so the largest magnitude lands
    at the top of the e4m3 range, and codes = e4m3(x / descale) (round to nearest even,
    computed in fp32).  The values the codes stand for are codes * descale."""
    amax = float(x.abs().max())
    descale = float(torch.tensor(amax / 448.0 if amax > 0 else 1.0, dtype=torch.float32))
    codes = (x.to(torch.float32) / torch.tensor(descale, dtype=torch.float32)).to(torch.float8_e4m3fn)
    return codes, descale


def make_inputs_e4m3(B: int, H: int, N: int, d: int, seed: int, *, H_kv: int | None = None) -> dict:
    """fp8 inputs: the fp32 normals of ``make_inputs`` (same generator order) quantised per
    tensor with ``quantize_e4m3``.  Returns codes ``q, k, v`` (torch.float8_e4m3fn) and their
    factors ``q_descale, k_descale, v_descale`` (Python floats holding fp32 values)."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(int(seed))
    hkv = H if H_kv is None else int(H_kv)
    out = {}
    for name in ("q", "k", "v"):
        heads = hkv if name in ("k", "v") else H
        out[name], out[name + "_descale"] = quantize_e4m3(
            torch.randn((B, N, heads, d), generator=gen, dtype=torch.float32))
    return out


def make_workload_inputs(w: Workload) -> dict[str, torch.Tensor]:
    if w.dtype == "e4m3":
        return make_inputs_e4m3(w.B, w.H, w.N, w.d, w.seed, H_kv=w.H_kv)
    return make_inputs(w.B, w.H, w.N, w.d, w.seed, with_do=w.backward, peaked=w.peaked, H_kv=w.H_kv,
                       dtype=w.torch_dtype)


def sample_rows(N: int, count: int | None, seed: int) -> torch.Tensor:
    """Sorted distinct rows in [0, N): a seeded sample of ``count`` plus {0, 1, N-1}.

    ``count=None`` (or count >= N) returns every row.
    """
    if count is None or count >= N:
        return torch.arange(N, dtype=torch.int64)
    gen = torch.Generator(device="cpu")
    gen.manual_seed(int(seed))
    picked = torch.randperm(N, generator=gen)[:count]
    fixed = torch.tensor([0, min(1, N - 1), N - 1], dtype=torch.int64)
    return torch.unique(torch.cat([picked, fixed]))


def head_row_seed(w_seed: int, b: int, h: int) -> int:
    """Per-(batch, head) seed for row sampling."""
    return int(w_seed) * 1_000_003 + b * 1009 + h * 7 + 17
