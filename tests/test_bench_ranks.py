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


def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference` (the fp64 oracle on the host cores) prints one JSON line
    with the contract's keys; it needs no GPU."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference",
                          "--config", "0", "--steps", "1", "--warmup", "3"],
                         check=True, capture_output=True, text=True, timeout=600).stdout
    lines = [ln for ln in out.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["value"] > 0 and j["unit"] == "query-tokens/s"
    for key in ("metric", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in j, key
    assert j["steps"] == 1 and j["warmup"] == 3 and j["higher_is_better"] is True
    assert j["cpu_baseline"]["kind"] == "oracle" and j["cpu_baseline"]["value"] == j["value"]
    assert j["e2e"] == {"value": j["value"], "unit": j["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
