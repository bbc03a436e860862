"""Multi-rank plumbing of bench.py on CPU: two gloo ranks, replicas timing.

bench.py runs one independent replica per GPU (no data-path collective) and
reports the slowest rank's time and the units of all ranks; this checks that
reduction with world size 2 on the gloo backend.
"""
from __future__ import annotations

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    ms, units = bench.reduce_over_ranks(10.0 + 5.0 * rank, 100.0, world)
    q.put((rank, ms, units))
    dist.barrier()
    dist.destroy_process_group()


def test_replicas_reduce_takes_slowest_rank_and_sums_units():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert out == [(0, 15.0, 200.0), (1, 15.0, 200.0)]


def test_single_rank_is_identity():
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    assert bench.reduce_over_ranks(3.5, 7.0, 1) == (3.5, 7.0)
