"""Multi-process host logic, on CPU with gloo (world size 2).

The benchmark shards by rows with no data-path collective; what crosses ranks is the
barrier and the max-over-ranks time.  The tensor-parallel all-reduce + add_rms_norm
gathers every rank's partial output in rank order before the fused kernel; here the
kernel is stood in for by the oracle (CPU tensors), which checks the gather, the order
and that every rank computes the same result.  A rank that leaves between steps makes the
remaining rank's next gather fail (short process-group timeout) instead of hanging.
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


def _tp_worker(rank, world, port, out):
    import numpy as np
    import oracle
    from rope_add_rms_b200 import synth, tp
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        inp = synth.allreduce_inputs(6, 32, world, "f32", seed=3)
        seen = {}

        def fake_kernel(parts, r, w, y, h, eps, x_out=None, stream=None):
            seen["parts"] = [p.clone() for p in parts]
            yy, hh, _ = oracle.allreduce_add_rms_norm([p.numpy() for p in parts], r.numpy(),
                                                      w.numpy(), eps)
            y.copy_(torch.from_numpy(yy.astype(np.float32)))
            h.copy_(torch.from_numpy(hh))

        tp.nv_allreduce_add_rms_norm = fake_kernel
        y, h = tp.allreduce_add_rms_norm(inp["parts"][rank], inp["r"], inp["w"], 1e-5)
        for i, p in enumerate(seen["parts"]):
            assert torch.equal(p, inp["parts"][i]), f"part {i} is not rank {i}'s partial"
        out[rank] = (y.numpy().tobytes(), h.numpy().tobytes())
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_tp_allreduce_gathers_in_rank_order_two_processes():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_tp_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    assert res[0] == res[1], "every rank must compute the same y and h"


def _leaving_worker(rank, world, port, out):
    import datetime
    import time
    from rope_add_rms_b200 import tp
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=5))
    dist.barrier()              # one step completes on every rank
    if rank == 1:
        os._exit(0)             # rank 1 leaves between steps, with nothing in flight
    t0 = time.monotonic()
    try:
        tp.gather_parts(torch.ones(4, 8))
        out[rank] = ("no error", time.monotonic() - t0)
    except Exception as e:  # noqa: BLE001 -- the error is what is checked
        out[rank] = (type(e).__name__, time.monotonic() - t0)
    finally:
        try:
            dist.destroy_process_group()
        except Exception:  # noqa: BLE001
            pass


def test_a_rank_that_leaves_ends_the_next_gather_with_an_error():
    """A rank that leaves between steps: the remaining rank's next gather of the partial
    outputs ends with an error within the process group's short timeout, not a hang."""
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_leaving_worker, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        hung = [p for p in procs if p.is_alive()]
        for p in hung:
            p.kill()
            p.join()
        res = dict(out)
    assert not hung, "a rank is still waiting in its collective"
    name, took = res[0]
    print(f"remaining rank: {name} after {took:.2f} s")
    assert name != "no error", "the gather with a departed rank must fail"
    assert took < 60
