"""The benchmark's multi-rank plumbing on CPU with the gloo backend (world size 2): the max
over ranks of the timed durations, the whole-job throughput, and the reference arm's
rank-0-only output. The layer itself does not shard (replicas only)."""
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = [10.0 + rank, 50.0 - 7 * rank]
        got = bench.reduce_max(mine, world, "cpu")
        results[rank] = got
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_reduce_max_two_ranks():
    world, port = 2, _free_port()
    with mp.Manager() as m:
        results = m.dict()
        mp.spawn(_worker, args=(world, port, results), nprocs=world, join=True)
        assert results[0] == results[1] == [11.0, 50.0]


def test_throughput_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench
    # 2 ranks x 10 steps x 4096 tokens in 5 ms (the slowest rank) -> 16.384 M tokens/s
    assert bench.tokens_per_second(4096, 10, 2, 5.0) == pytest.approx(16.384e6)
    assert bench.reduce_max([1.0, 2.0], 1, "cpu") == [1.0, 2.0]


def test_reference_arm_prints_only_on_rank_0():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], capture_output=True, text=True, env=env,
                       timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""
