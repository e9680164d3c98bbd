"""Replica bookkeeping for multi-GPU benchmark runs (no attention arithmetic).

Every (batch, head) of exact attention is independent and the method has no exchange
step, so N GPUs run N independent replicas of the same workload: weak scaling, no
data-path collective.  The only cross-rank traffic is timing: each rank measures its own
device time and the job time is the maximum over ranks.
"""
from __future__ import annotations

import os

import torch


def world() -> tuple[int, int, int]:
    """(world_size, rank, local_rank) from the launcher's environment (1, 0, 0 without one)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(values, device: torch.device | str = "cpu") -> list[float]:
    """Element-wise maximum of per-rank values across the default process group."""
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def whole_job_tflops(world_size: int, flops_per_rank_step: float, ms_per_step_max: float) -> float:
    """Aggregate TFLOP/s of all replicas: every rank does the same work per step."""
    return world_size * flops_per_rank_step / (ms_per_step_max * 1e-3) / 1e12
