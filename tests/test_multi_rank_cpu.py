"""The multi-process plumbing of bench.py on CPU: two gloo ranks, the
maximum-over-ranks timing and the whole-job (weak-scaling) throughput."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    assert bench.dist_env() == (world, rank, rank)
    seconds = [0.25, 0.5][rank]            # rank 1 is the slow one
    slowest = bench.reduce_max(seconds, world)
    out[rank] = (slowest, bench.weak_value(1000.0, world, slowest))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    world, port = 2, _free_port()
    out = mp.Manager().dict()
    mp.spawn(_rank, args=(world, port, out), nprocs=world, join=True)
    for r in range(world):
        slowest, value = out[r]
        assert slowest == pytest.approx(0.5)
        assert value == pytest.approx(2 * 1000.0 / 0.5)


def test_single_rank_is_identity():
    import bench
    assert bench.reduce_max(1.25, 1) == 1.25
    assert bench.weak_value(10.0, 1, 2.0) == 5.0
