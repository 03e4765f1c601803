"""Host logic of bench.py's multi-rank path, on CPU ranks over gloo.

With N > 1 every rank times its own copy of the workload, the step time is the
maximum over ranks (all_reduce MAX), and the reported value counts the units of
every rank. The reference arm prints from rank 0 only.
"""

import json
import os
import socket
import subprocess
import sys
from datetime import timedelta

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, per_rank_ms, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist

    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        ms_max = bench._max_over_ranks(per_rank_ms[rank], world, torch.device("cpu"))
        bench._barrier(world)
        value = bench.whole_job_rate(1000, 4, world, ms_max)
        out.put((rank, ms_max, value))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_max_over_ranks_and_whole_job_value(world):
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    per_rank_ms = [10.0, 25.0][:world]
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, per_rank_ms, out))
             for r in range(world)]
    for p in procs:
        p.start()
    got = [out.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    expect_ms = max(per_rank_ms)
    for rank, ms_max, value in got:
        assert ms_max == expect_ms  # every rank sees the slowest rank's time
        # units of all ranks over the slowest rank's time
        assert value == pytest.approx(1000 * 4 * world / (expect_ms / 1e3))


def test_whole_job_rate_single_rank():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.whole_job_rate(2048, 10, 1, 5.0) == pytest.approx(2048 * 10 / 5e-3)


def test_reference_arm_prints_from_rank0_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0", "--workload", "fp32_small"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_reference_arm_rank0_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "2", "--warmup", "1", "--workload", "fp32_small"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["value"] > 0
