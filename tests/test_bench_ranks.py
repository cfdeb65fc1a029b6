"""The benchmark's multi-rank host logic on the CPU (two processes, no GPU).

The path has no data-path collective: ranks are independent replicas, and the only
cross-rank step is the timing rule (every multi-rank time is the slowest rank's).
Covered here: that reduction over a world-size-2 gloo group, and the reference arm
launched under torchrun with two ranks (rank 0 alone runs and prints one line).
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, results):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r took (r + 1) * 1.5 ms: both ranks must report the slower one
        results[rank] = bench.max_over_ranks((rank + 1) * 1.5, world, "cpu")
    finally:
        dist.destroy_process_group()


def test_time_is_the_slowest_rank_over_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), results), nprocs=world, start_method="spawn",
                           join=True)
        assert dict(results) == {0: 3.0, 1: 3.0}


def test_single_rank_time_is_its_own():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(2.25, 1, "cpu") == 2.25


@pytest.mark.slow
def test_reference_arm_under_torchrun_two_ranks():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           "bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
