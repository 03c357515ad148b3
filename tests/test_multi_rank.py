"""Host logic of the multi-GPU launch on CPU ranks (gloo, world size 2).

The path has no exchange step: with N GPUs `bench.py` runs N independent
replicas, times each on its own device, takes the slowest rank's time and
reports the whole job's throughput from rank 0.  These tests run that
reduction on two gloo ranks, and check that only rank 0 of a multi-rank
launch runs the CPU reference arm."""
import multiprocessing as mp
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    ms = bench.max_over_ranks(times[rank], dist, "cpu")
    rate = bench.job_rate(1e9, world, ms)
    dist.barrier()
    dist.destroy_process_group()
    out.put((rank, ms, rate))


def test_max_over_ranks_and_job_rate_on_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    times = [12.5, 20.0]  # rank 1 is the slow one
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, times, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, rate in res:
        assert ms == 20.0                          # every rank sees the slowest time
        assert rate == pytest.approx(2 * 1e9 / 20e-3)  # both replicas' units / that time


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25, None, "cpu") == 3.25
    assert bench.job_rate(10.0, 1, 1000.0) == pytest.approx(10.0)


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "1"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""
