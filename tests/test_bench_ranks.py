"""bench.py's replica plumbing on CPU: two ranks over gloo (127.0.0.1) take
the same collective steps; the timed region of the job is the slowest rank's
(max over ranks, seen by every rank), and the barrier releases only when both
ranks have arrived."""
import os
import socket
import sys
import time

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # rank 1 arrives late: the barrier must hold rank 0 until then
        if rank == 1:
            time.sleep(0.5)
        t0 = time.time()
        bench.barrier(world)
        waited = time.time() - t0
        dt = bench.max_over_ranks(1.0 + rank * 2.5, world)
        q.put((rank, waited, dt))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_barrier_and_max():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, w0, d0), (r1, w1, d1) = res
    assert (r0, r1) == (0, 1)
    assert w0 >= 0.3                      # rank 0 waited for rank 1
    assert d0 == d1 == 3.5                # both ranks see the slowest time


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(2.25, 1) == 2.25
    bench.barrier(1)
