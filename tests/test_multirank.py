"""The benchmark's multi-process path on the CPU: one gloo process per rank, as
torchrun would start them. The hot path has no exchange step (ranks are
independent replicas), so what is checked is the timing aggregation: every
rank agrees on the slowest rank's time and the whole-job rate is the units of
all ranks over that time; the reference arm prints only on rank 0."""
import os
import socket
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        slowest = bench.max_over_ranks(times[rank])
        rate = bench.job_throughput(1000.0, world, slowest)
        out[rank] = (slowest, rate)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_max_over_ranks_and_job_rate(world):
    times = [0.5 + 0.25 * r for r in range(world)][::-1]  # rank 0 is the slowest
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), times, out), nprocs=world, join=True)
        results = dict(out)
    slowest = max(times)
    for r in range(world):
        assert results[r][0] == slowest
        assert results[r][1] == pytest.approx(world * 1000.0 / slowest)


def test_single_process_is_identity():
    assert bench.max_over_ranks(1.25) == 1.25
    assert bench.job_throughput(10.0, 1, 2.0) == 5.0


def test_reference_arm_prints_only_on_rank_zero():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "3",
                          "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert res.returncode == 0 and res.stdout.strip() == ""
