"""The multi-GPU path is "replicas only": each rank runs an independent copy
of the step, and the job's time is the slowest rank's.  These tests exercise
bench.py's barrier and max-over-ranks plumbing with world_size 2 on CPU
(gloo), and the whole-job throughput arithmetic."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    ctx = bench.DistCtx(backend="gloo", timeout_s=60)
    ctx.barrier()
    # rank-dependent "measured" per-case times
    got = ctx.max_over_ranks([1.0 + rank, 10.0 - rank, 0.5 * rank])
    ctx.barrier()
    results[rank] = got
    ctx.close()


def test_max_over_ranks_gloo_world2():
    world = 2
    with mp.Manager() as m:
        results = m.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), results), nprocs=world, join=True)
        assert results[0] == results[1] == [2.0, 10.0, 0.5]


def test_aggregate_throughput_is_sum_over_replicas_at_slowest_time():
    import bench
    # 2 replicas, each 1e12 FLOP, slowest took 1 ms -> 2000 TFLOP/s
    assert bench.aggregate_throughput(1e12, 1.0, 2, 1e12) == pytest.approx(2000.0)
    assert bench.aggregate_throughput(4e9, 2.0, 1, 1e9) == pytest.approx(2000.0)
