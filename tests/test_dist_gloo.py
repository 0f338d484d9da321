"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): max-over-ranks timing and
per-rank request shards (weak scaling, no collective on the data path)."""

import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import torch.distributed as dist
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    from workloads import WORKLOADS, draw_seqlens
    t = bench.reduce_max(0.5 + rank * 0.25)
    w = WORKLOADS["varlen-mtp"]
    g = torch.Generator().manual_seed(bench.shard_seed(w.seed, rank))
    lens = draw_seqlens(w, g)
    out[rank] = (t, bench.shard_seed(w.seed, rank), sum(lens), len(lens))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_max_and_shards():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    port = _free_port()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    assert out[0][0] == out[1][0] == 0.75, "elapsed time must be the max over ranks"
    assert out[0][1] != out[1][1], "ranks must draw different shards"
    assert out[0][3] == out[1][3] == 132, "each rank runs a full batch (weak scaling)"
    assert out[0][2] != out[1][2]


def test_single_process_reduce_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(1.25) == 1.25
    assert bench.shard_seed(1003, 0) == 1003
