"""The N > 1 bench path on CPU: two gloo ranks, as torchrun starts them.

With several GPUs every rank runs an independent replica of the layer (the
pass has no exchange step); the job's time is the slowest rank's, which
every rank receives, and the job's throughput counts every replica. These
are the two host-side steps of that path, run here over a world of two
processes on the gloo backend (no GPU)."""

import os
import socket

import pytest
import torch.multiprocessing as tmp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, results):
    import datetime

    import torch
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, dist, torch.device("cpu"))
        value = bench.job_throughput(world, 2.0e12, ms)
        results[rank] = (ms, value)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_count_both_replicas():
    port = _free_port()
    with tmp.Manager() as m:
        results = m.dict()
        tmp.spawn(_rank, args=(2, port, results), nprocs=2, join=True)
        got = dict(results)
    assert sorted(got) == [0, 1]
    for ms, value in got.values():
        assert ms == 15.0                       # the slower rank's time on both ranks
        assert value == pytest.approx(2 * 2.0e12 / 15.0e-3 / 1e12)


def test_one_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(12.5, None, None) == 12.5
    assert bench.job_throughput(1, 107.87e12, 46.84) == pytest.approx(107.87e12 / 46.84e-3 / 1e12)
