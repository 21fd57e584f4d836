"""The multi-GPU bench path on CPU: two gloo ranks agree on the slowest rank's
time and the whole-job throughput counts every rank's work once."""
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        mine = [120.0, 135.5][rank]               # per-rank timed milliseconds
        mx = bench.max_over_ranks(mine, world)
        q.put((rank, mx, bench.aggregate_tops(world, 1.4e14, 10, mx)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_count_all_work():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert res[0][1] == res[1][1] == 135.5
    expect = 2 * 1.4e14 * 10 / 0.1355 / 1e12
    assert abs(res[0][2] - expect) < 1e-9 * expect


def test_single_rank_is_identity():
    assert bench.max_over_ranks(7.5, 1) == 7.5
    assert abs(bench.aggregate_tops(1, 1e12, 1, 1000.0) - 1.0) < 1e-12


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--steps", "1", "--warmup", "0"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""
