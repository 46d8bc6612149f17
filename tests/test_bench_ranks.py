"""Multi-rank timing logic of bench.py on CPU: two gloo ranks, each with its own
timings, agree on the element-wise maximum (the job runs as long as its slowest
rank), and a single rank keeps its own values."""
import os
import socket
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = [1.0 + rank, 10.0 - rank, 3.5 * (rank + 1)]
        out[rank] = bench.max_over_ranks(mine, dist, "cpu")
    finally:
        dist.destroy_process_group()


def test_max_over_two_gloo_ranks():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(world, _free_port(), out), nprocs=world, join=True)
        got = dict(out)
    assert got[0] == got[1] == [2.0, 10.0, 7.0]


def test_single_rank_keeps_its_values():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([3, 1.5]) == [3.0, 1.5]
