"""Multi-process host logic of the benchmark, on CPU with gloo (world size 2).

The path shards by rows with no data-path collective; what crosses ranks is the
barrier and the max-over-ranks time.  These tests run that logic in two processes.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, times, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        r, w, lr = bench.dist_env()
        assert (r, w, lr) == (rank, world, rank)
        got = bench.max_over_ranks(times[rank], device="cpu")
        out[rank] = got + [bench.shard_seed(rank)]
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_shards_two_processes():
    world = 2
    times = [[41.0, 5000.0], [43.5, 4900.0]]
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, _free_port(), times, out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        assert res[rank][:2] == [43.5, 5000.0], "every rank sees the slowest rank's times"
    assert res[0][2] != res[1][2], "ranks draw different rows"


def test_single_process_is_identity_and_throughput_formula():
    assert bench.max_over_ranks([1.0, 2.0], device="cpu") == [1.0, 2.0]
    # two ranks, 268,443,648 bytes per step, 1000 steps, slowest rank 41.79 ms in total
    v = bench.job_throughput(2, 268443648, 1000, 41.79)
    assert v == pytest.approx(2 * 268443648 * 1000 / 0.04179 / 1e9)
