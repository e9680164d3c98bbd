"""The multi-rank host logic of the benchmark, run as two gloo ranks on CPU."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from exact_io_aware_93_b200.replicas import whole_job_tflops


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world_size, port, out):
    import torch.distributed as dist
    from exact_io_aware_93_b200.replicas import max_over_ranks, world
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world_size), "LOCAL_RANK": str(rank)})
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world_size,
                            timeout=datetime.timedelta(seconds=60))
    try:
        assert world() == (world_size, rank, rank)
        # rank r "measured" 1.0 + r ms per step and 10 + 5r ms end to end
        mx = max_over_ranks([1.0 + rank, 10.0 + 5 * rank, 0.5 * (2 - rank)])
        out[rank] = mx
    finally:
        dist.destroy_process_group()


def test_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == out[1] == [2.0, 15.0, 1.0]


def test_whole_job_value_is_weak_scaling_aggregate():
    assert whole_job_tflops(1, 1e12, 1.0) == pytest.approx(1000.0)
    assert whole_job_tflops(4, 1e12, 2.0) == pytest.approx(2000.0)


def test_max_over_ranks_single_process():
    from exact_io_aware_93_b200.replicas import max_over_ranks
    assert max_over_ranks([3.0, 1.5]) == [3.0, 1.5]
