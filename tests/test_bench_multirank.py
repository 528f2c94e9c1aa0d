"""The bench's multi-rank host logic on CPU with the gloo backend (two ranks):
the timed region is the slowest rank's, the value is the whole job's, and the
reference arm runs on rank 0 only."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # each rank's own step time; the job's is the largest
        elapsed = bench.ranks_max(100.0 + 25.0 * rank, dist, "cpu")
        out[rank] = (elapsed, bench.whole_job_rate(world, 1000, 4, elapsed))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_the_whole_job_value():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    assert res[0] == res[1]
    elapsed, value = res[0]
    assert elapsed == 125.0
    assert value == pytest.approx(2 * 1000 * 4 / 0.125)


def test_single_process_needs_no_group():
    import bench
    assert bench.ranks_max(3.5, None, "cpu") == 3.5
    assert bench.whole_job_rate(1, 10, 2, 1000.0) == pytest.approx(20.0)


def _run_reference(env_extra):
    env = dict(os.environ, **env_extra)
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
           "--config", "tiny_f32", "--steps", "1", "--warmup", "0"]
    return subprocess.run(cmd, env=env, capture_output=True, text=True, timeout=600)


def test_reference_arm_runs_on_rank_zero_only():
    r1 = _run_reference({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    r0 = _run_reference({"RANK": "0", "WORLD_SIZE": "1", "LOCAL_RANK": "0"})
    assert r0.returncode == 0, r0.stderr[-2000:]
    lines = [x for x in r0.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
