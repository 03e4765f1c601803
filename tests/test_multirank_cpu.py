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


def _sp_rank_main(rank, world, port, out):
    """One rank of a sequence split in `world` parts: the exchange of
    linear_attention_la2_b200.sp over gloo, with the float64 oracle standing in
    for the kernels (la2_kv_state -> oracle.kv_state, la2_forward_sp ->
    oracle.forward_from_state)."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist

    import oracle
    from linear_attention_la2_b200 import sp

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        g = torch.Generator().manual_seed(123)  # every rank draws the whole sequence
        B, H, N, d = 1, 2, 60, 4
        q, k, v, do = (torch.randn((B, H, N, d), generator=g, dtype=torch.float64) for _ in range(4))
        a, b = N * rank // world, N * (rank + 1) // world
        sl = (slice(None), slice(None), slice(a, b))
        local = torch.from_numpy(oracle.kv_state(k[sl], v[sl]))
        kv = sp.exchange_states(local)
        before, after = sp.prefix_suffix(kv, rank)
        o = oracle.forward_from_state(q[sl], k[sl], v[sl], before.sum(0).numpy())
        qdo = sp.exchange_states(torch.from_numpy(oracle.kv_state(q[sl], do[sl])))
        _, later = sp.prefix_suffix(qdo, rank)
        gq, gk, gv = oracle.backward_from_states(q[sl], k[sl], v[sl], do[sl], before.sum(0).numpy(),
                                                 later.sum(0).numpy())
        whole = oracle.forward(q, k, v, True)[:, :, a:b]
        wq, wk, wv = (x[:, :, a:b] for x in oracle.backward(q, k, v, do, True))
        err = max(float(abs(o - whole).max()), float(abs(gq - wq).max()), float(abs(gk - wk).max()),
                  float(abs(gv - wv).max()))
        out.put((rank, kv.shape[0], before.shape[0], after.shape[0], err))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sequence_parallel_exchange(world):
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_sp_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted(out.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, gathered, n_before, n_after, err in got:
        assert gathered == world and n_before == rank and n_after == world - 1 - rank
        assert err < 1e-10
