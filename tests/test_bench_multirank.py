"""The multi-rank host logic of bench.py on CPU: two gloo ranks.

Each rank reports its own step time; every rank must end up with the slowest
one (the whole job is as fast as its slowest rank), the job throughput counts
every rank's work, and the reference arm only runs on rank 0.
"""
import io
import os
import sys
from contextlib import redirect_stdout

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = 10.0 + 5.0 * rank  # rank 1 is the slow one
        got = bench.max_over_ranks(mine, dist, torch.device("cpu"))
        value = bench.job_throughput(1e12, world, got)
        with open(os.path.join(out_dir, f"r{rank}.txt"), "w") as fh:
            fh.write(f"{got} {value}\n")
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput(tmp_path):
    world, port = 2, 29611
    mp.start_processes(_worker, args=(world, port, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    for r in range(world):
        got, value = (float(x) for x in open(tmp_path / f"r{r}.txt").read().split())
        assert got == 15.0
        assert abs(value - 2 * 1e12 / 15e-3 / 1e12) < 1e-9


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")

    class Args:
        steps, warmup = 1, 0

    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(Args(), bench.SI.TINY)
    assert buf.getvalue() == ""


@pytest.mark.slow
def test_reference_arm_prints_one_line_on_rank_zero(monkeypatch):
    import json
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("WORLD_SIZE", "1")
    monkeypatch.setenv("RANK", "0")

    class Args:
        steps, warmup = 1, 0

    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(Args(), bench.SI.TINY)
    lines = buf.getvalue().strip().splitlines()
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["e2e"]["h2d_bytes_per_step"] == 0
