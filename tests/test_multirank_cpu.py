"""The N > 1 host path of bench.py on CPU ranks (gloo, world size 2): each rank
gets its own shard of the global batch, and timings reduce to the max over ranks."""
from __future__ import annotations

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    from io_aware_exact_23_b200.inputs import TINY, make_inputs
    w = bench.rank_workload(TINY, rank)
    t = make_inputs(w)
    # every rank reports different times; all must agree on the max
    got = bench.reduce_max([1.0 + rank, 10.0 - rank, 3.0], dist, torch.device("cpu"))
    h = float(t["q"].float().sum())
    hs = [None] * world
    dist.all_gather_object(hs, h)
    out[rank] = (got, w.seed, hs)
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks():
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()  # no fork of this (multi-threaded) test process
    out = mgr.dict()
    mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
    for r in range(2):
        got, seed, hs = out[r]
        assert got == [2.0, 10.0, 3.0]
        assert seed == r
        assert hs[0] != hs[1]  # the ranks hold different shards


def test_single_rank_reduce_is_identity():
    import bench
    assert bench.reduce_max([1.5, 2.5], None, torch.device("cpu")) == [1.5, 2.5]
