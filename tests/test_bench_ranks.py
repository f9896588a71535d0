"""Host logic of the multi-rank benchmark on CPU: two gloo ranks, each with its own step
times; every rank must see the maximum over ranks (the slowest replica sets the job time)."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        local = [1.0 + rank, 10.0 - rank, 0.5 * (rank + 1)]
        got = bench.combine_over_ranks(local, world, torch.device("cpu"))
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_combine_over_ranks_takes_the_max_on_every_rank():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
    for r in range(world):
        assert out[r] == [2.0, 10.0, 1.0]


def test_combine_over_ranks_single_rank_is_identity():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.combine_over_ranks([3.0, 4.5], 1, None) == [3.0, 4.5]


def test_fused_flop_count():
    import sys
    sys.path.insert(0, ROOT)
    import bench

    class W:
        N1, D, K, T1 = 64, 128, 2048, 4096
    assert bench.fused_algorithmic_flop(W, "keymajor") == 4.0 * 64 * 128 * 2048 * 4096
    assert bench.fused_algorithmic_flop(W, "scatter") == 6.0 * 64 * 128 * 2048 * 4096
