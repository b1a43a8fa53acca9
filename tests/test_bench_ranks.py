"""Host logic of the multi-GPU bench (replicas only) on CPU: two gloo ranks reduce their
timings to the max over ranks, and the whole-job rate counts every rank's work over the
slowest rank's time. Also: the reference arm does no work on ranks other than 0."""
from __future__ import annotations

import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 100.0 + 25.0 * rank           # rank 1 is the slow one
        dist.barrier()
        m = bench.reduce_max(local_ms, world)
        rate = bench.job_rate_tbs(world, 10, 1e9, m)
        q.put((rank, m, rate))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_time():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [r[1] for r in res] == [125.0, 125.0]                    # both ranks see the slowest rank
    assert res[0][2] == pytest.approx(2 * 10 * 1e9 / 0.125 / 1e12)  # work of both ranks / max time


def test_single_rank_reduction_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(3.5, 1) == 3.5
    assert bench.job_rate_tbs(1, 4, 2e12, 1000.0) == pytest.approx(8.0)


def test_reference_arm_is_silent_on_other_ranks():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0", "--workload", "tiny_f32"], capture_output=True, text=True, env=env,
                       timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
