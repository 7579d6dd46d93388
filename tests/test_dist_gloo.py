"""The multi-rank host logic of bench.py on CPU with the gloo backend (world size 2):
timing is the max over ranks and every rank draws its own batch rows."""
from __future__ import annotations

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks([10.0 + rank, 5.0 - rank])
        seeds = [bench.replica_seed(rank, l) for l in range(4)]
        gathered = [None] * world
        dist.all_gather_object(gathered, seeds)
        out[rank] = (got, gathered)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_distinct_seeds():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for r in range(world):
        got, gathered = res[r]
        assert got == [11.0, 5.0]
        flat = [s for per in gathered for s in per]
        assert len(set(flat)) == len(flat)


def test_single_process_identity():
    import bench
    assert bench.max_over_ranks([3.0, 4.0]) == [3.0, 4.0]
