"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2).

The decode path shards by sequence and needs no collective: ranks run
independent replicas, and only the timing is combined (max over ranks).  These
tests exercise that combination and the reference arm's rank handling without
a GPU.
"""
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


def _worker(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [0.8, 1.3][rank]
        got = bench.max_over_ranks(local_ms)
        dist.barrier()
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    mp.start_processes(_worker, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
    assert out[0] == out[1] == 1.3


def test_whole_job_rate_uses_slowest_rank():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.whole_job_tokens_per_s(1, 64, 0.8) == pytest.approx(80000.0)
    assert bench.whole_job_tokens_per_s(4, 64, 1.0) == pytest.approx(256000.0)
    assert bench.max_over_ranks(0.5) == 0.5          # not distributed: identity


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""
