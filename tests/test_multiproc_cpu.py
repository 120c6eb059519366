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


def _peer_worker(rank, world, port, out):
    """PeerAllReduce's host protocol on CPU: the device calls are fakes that record what
    they are given."""
    import datetime
    from rope_add_rms_b200 import tp
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        calls = []
        fake_base = {r: 0x7000_0000_0000 + (r << 32) for r in range(world)}  # peers' mappings

        def export(t):
            calls.append(("export", t.data_ptr(), t.numel()))
            return (f"handle-of-rank-{rank}".encode().ljust(64, b"\0"), 0)

        def imp(handle, offset):
            peer = int(handle.rstrip(b"\0").decode().rsplit("-", 1)[1])
            calls.append(("import", peer, offset))
            return fake_base[peer] + offset

        lib = {"export": export, "import": imp,
               "publish": lambda ptrs, rk, ep, stream=None: calls.append(("publish", list(ptrs), rk, ep)),
               "reduce": lambda parts, r, w, y, h, eps, flags, ep, stream=None:
                   calls.append(("reduce", list(parts), flags.data_ptr(), ep)),
               "close": lambda ptr, off: calls.append(("close", ptr, off))}
        shape = (6, 32)
        par = tp.PeerAllReduce(shape, torch.bfloat16, device="cpu", lib=lib)
        slots = []
        for step in range(3):
            slots.append(par.partial().data_ptr())
            par(torch.zeros(shape, dtype=torch.bfloat16), None, 1e-5)
        par.close()
        out[rank] = (calls, par.raw.data_ptr(), par.slot_bytes, par.flags_off, slots,
                     int(par.flags.abs().sum()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_peer_allreduce_host_protocol_two_processes():
    """Handles exchanged once in rank order (own memory used directly, each peer mapped
    once and closed at the end); per step the epoch grows by one, is published into every
    rank's flag slot before the reduction runs, and the parts are the epoch's slot of every
    rank's buffer in rank order, the slots alternating between steps (double buffering)."""
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_peer_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        calls, own, slot_bytes, flags_off, slots, flag_sum = res[rank]
        peer = 1 - rank
        peer_base = 0x7000_0000_0000 + (peer << 32)
        assert flag_sum == 0, "flags start at zero"
        assert slot_bytes == 6 * 32 * 2 and flags_off >= 2 * slot_bytes
        assert [c[0] for c in calls[:2]] == ["export", "import"] and calls[1][1] == peer
        bases = {rank: own, peer: peer_base}
        steps = [c for c in calls if c[0] in ("publish", "reduce")]
        assert [c[0] for c in steps] == ["publish", "reduce"] * 3
        for i in range(3):
            pub, red = steps[2 * i], steps[2 * i + 1]
            epoch = i + 1
            assert pub[3] == epoch and red[3] == epoch and pub[2] == rank
            assert pub[1] == [bases[r] + flags_off for r in range(world)]
            assert red[1] == [bases[r] + (epoch & 1) * slot_bytes for r in range(world)]
            assert red[2] == own + flags_off, "the reduction waits on this rank's own flags"
            assert slots[i] == own + (epoch & 1) * slot_bytes, "partial() is this step's slot"
        assert calls[-1] == ("close", peer_base, 0)
