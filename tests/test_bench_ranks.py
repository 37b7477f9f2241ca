"""Host-side logic of bench.py's multi-GPU (replica) path, on CPU: two gloo
ranks take the maximum of their timings, the job throughput counts every
rank's bytes, and the reference arm prints on rank 0 only."""
from __future__ import annotations

import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, q) -> None:
    import datetime

    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r measured (1 + r) ms for the kernel loop and 10 (1 + r) ms end to end
        ms, ms_e2e = bench.max_over_ranks([1.0 + rank, 10.0 * (1 + rank)], dist, "cpu")
        q.put((rank, ms, ms_e2e, bench.job_gbs(world, 1000, 500, ms)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, ms, ms_e2e, gbs in got:
        assert ms == 2.0 and ms_e2e == 20.0  # every rank sees the slowest rank's times
        assert gbs == pytest.approx(2 * 1000 * 500 / 2e-3 / 1e9)


def test_single_process_timing_is_unchanged():
    assert bench.max_over_ranks([3.5, 7.0], None, "cpu") == [3.5, 7.0]
    assert bench.job_gbs(1, 30507008, 100, 1.2) == pytest.approx(30507008 * 100 / 1.2e-3 / 1e9)


def test_reference_arm_prints_on_rank0_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "0", "--cpu-budget", "0.2"], env=env, capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip() == ""
