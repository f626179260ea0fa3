"""Failure detection across ranks, on the host (gloo, CPU): a rank that exits
between steps, with nothing in flight, must make the next collective of the
others end with an error instead of waiting for ever.  The bench's own
collective helpers (barrier, max over ranks) are the ones exercised; the
process group is given a short timeout as the last bound."""
import datetime
import os
import socket
import sys
import time

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, which, out_q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=20))
    bench.barrier(world)  # one step completed together
    if rank == world - 1:
        os._exit(3)  # this rank dies between steps, without leaving the group
    t0 = time.time()
    try:
        if which == "barrier":
            bench.barrier(world)
        else:
            bench.max_over_ranks(1.0, world)
        out_q.put((rank, "returned", time.time() - t0))
    except Exception as e:  # the expected outcome
        out_q.put((rank, type(e).__name__, time.time() - t0))
    out_q.close()
    out_q.join_thread()  # flush the queue's feeder thread before the hard exit
    os._exit(0)


def _run(world, which):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, which, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = [q.get(timeout=120) for _ in range(world - 1)]
    for p in procs:
        p.join(60)
    return got, [p.exitcode for p in procs]


def test_survivors_collective_errors_when_a_rank_dies():
    for world, which in ((2, "max"), (3, "barrier")):
        got, codes = _run(world, which)
        assert codes[-1] == 3
        for rank, outcome, dt in got:
            assert outcome != "returned", f"rank {rank}: the collective returned although a rank had died"
            assert dt < 60, f"rank {rank}: the error took {dt:.0f} s"


def _ulysses_rank_main(rank, world, port, out_q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import numpy as np
    import torch
    import torch.distributed as dist

    from exact_io_aware_sm_b200.ulysses import ulysses_attention
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=20))
    dist.barrier()
    if rank == world - 1:
        os._exit(3)
    x = torch.from_numpy(np.random.default_rng(rank).standard_normal((1, 8, 4, 8)))

    def att(q, k, v, mk, sc):  # never reached: the exchange before it fails
        raise AssertionError("attention ran without every rank's rows")
    t0 = time.time()
    try:
        ulysses_attention(x, x, x, attention=att, shard_lens=[8] * world)
        out_q.put((rank, "returned", time.time() - t0))
    except Exception as e:
        out_q.put((rank, type(e).__name__, time.time() - t0))
    out_q.close()
    out_q.join_thread()
    os._exit(0)


def test_ulysses_exchange_errors_when_a_rank_dies():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    world = 2
    procs = [ctx.Process(target=_ulysses_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = [q.get(timeout=120) for _ in range(world - 1)]
    for p in procs:
        p.join(60)
    for rank, outcome, dt in got:
        assert outcome not in ("returned", "AssertionError"), f"rank {rank}: {outcome}"
        assert dt < 60, f"rank {rank}: the error took {dt:.0f} s"
