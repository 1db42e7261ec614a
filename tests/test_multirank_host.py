"""The multi-rank plumbing of bench.py on CPU: two gloo ranks, disjoint samples, and the
max-over-ranks reduction that sets the job time."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local = 10.0 + 5.0 * rank
        out[rank] = (bench.max_over_ranks(local), list(bench.rank_samples(rank, 3)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_disjoint_samples():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:     # no fork of a threaded process
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0
    assert set(res[0][1]).isdisjoint(res[1][1])
    assert res[0][1] == [0, 1, 2] and res[1][1] == [3, 4, 5]


def test_single_process_max_is_local():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
