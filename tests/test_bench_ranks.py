"""Host logic of the multi-GPU bench path, on CPU ranks over gloo.

The decode path does not shard: each GPU serves its own independent sequences and no collective
touches the data.  What runs on more than one rank is the bench's bookkeeping -- every rank
reports its device time, the job's time is the slowest rank's, and the job's rate is the units
all ranks processed over that time -- and the reference arm, which only rank 0 runs.  Both are
exercised here with two spawned CPU processes (world size 2, gloo on 127.0.0.1)."""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as td
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    td.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(times[rank], "cpu")
        units = 8 * 30                                  # 8 sequences x 30 steps on every rank
        q.put((rank, ms, bench.job_throughput(units, ms, world)))
        td.barrier()
    finally:
        td.destroy_process_group()


@pytest.mark.parametrize("times", [(3.0, 5.0), (7.25, 2.0)])
def test_job_time_is_the_slowest_rank_and_rate_counts_every_rank(times):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, times, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    slowest = max(times)
    for _, ms, rate in res:
        assert ms == slowest
        assert rate == pytest.approx(world * 8 * 30 / (slowest * 1e-3))


def test_single_process_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert not td.is_initialized()
    assert bench.max_over_ranks(4.5, "cpu") == 4.5
    assert bench.job_throughput(240, 4.5, 1) == pytest.approx(240 / 4.5e-3)


def test_reference_arm_runs_on_rank_zero_only():
    """Under torchrun every rank starts the reference arm; ranks other than 0 must exit 0
    without work or output."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_profiled_traffic_is_dropped_once_the_kernel_changes(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    t = bench.profiled_traffic("indexer", "decode1m")
    if t is not None:
        assert t > 0
    monkeypatch.setattr(bench, "kernel_source_hash", lambda cu: "0000000000000000")
    assert bench.profiled_traffic("indexer", "decode1m") is None
    assert bench.profiled_traffic("indexer", "decode128k") is None
