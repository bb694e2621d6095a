"""World-size-2 checks of the multi-rank benchmark plumbing on CPU (gloo).

bench.py --gpus N runs N independent replicas (one process per GPU, its own histories): the only
exchanges are barriers and the max over ranks of the device-timed duration. Both are exercised
here with two gloo ranks on 127.0.0.1.
"""

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

    import torch
    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks(1.5 + rank * 2.25, torch.device("cpu"))
        dist.barrier()
        out[rank] = (got, bench.rank_seed(rank))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_max_over_ranks_and_distinct_seeds_two_ranks():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    assert out[0][0] == out[1][0] == 1.5 + 2.25
    assert out[0][1] != out[1][1]


def test_single_process_is_identity():
    import torch

    import bench
    assert bench.max_over_ranks(3.25, torch.device("cpu")) == 3.25


@pytest.mark.timeout(300)
def test_bench_gpus_two_launches_two_ranks():
    """`bench.py --gpus 2` (no torchrun around it) launches two ranks itself; the CPU dry run
    exercises the same launch, barriers and max-over-ranks timing, and rank 0 alone prints one
    line that reports the two ranks it ran."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    res = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2",
                          "--dry-run", "--steps", "2", "--warmup", "3"], cwd=root, env=env,
                         capture_output=True, text=True, timeout=280)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["n_gpus"] == 2 and line["ranks_timed"] == 2 and line["dry_run"] is True
