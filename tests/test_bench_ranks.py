"""Multi-rank bench logic on CPU (gloo, world size 2): the job's time is the
slowest rank's and its throughput counts every rank's sequences; under the
reference arm only rank 0 works and prints."""
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


def _rank_main(rank, world, port, local_ms, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        value, total_ms = bench.job_value(local_ms[rank], world, 64 * 10, dist)
        q.put((rank, value, total_ms))
    finally:
        dist.destroy_process_group()


def test_job_value_takes_the_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    local_ms = [10.0, 25.0]
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, local_ms, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, value, total_ms in got:
        assert total_ms == 25.0
        assert value == pytest.approx(2 * 64 * 10 / 0.025)


def test_job_value_single_rank():
    sys.path.insert(0, ROOT)
    import bench
    value, total_ms = bench.job_value(40.0, 1, 64 * 20)
    assert total_ms == 40.0 and value == pytest.approx(64 * 20 / 0.040)


def test_reference_arm_non_zero_rank_is_silent():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "3", "--warmup", "1"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""
