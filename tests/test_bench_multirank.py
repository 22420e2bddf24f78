"""Host logic of bench.py's multi-process path, run as two gloo ranks on CPU: the device-timed
step time is the maximum over ranks, the whole-job value counts every rank's work (weak scaling),
and the reference arm does its work on rank 0 only."""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, q):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(times[rank], dist, torch.device("cpu"))
        dist.barrier()
        q.put((rank, ms, bench.whole_job_tflops(world, ms)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_value_two_gloo_ranks():
    import bench
    world, port = 2, _free_port()
    times = [1.25, 0.75]                 # rank 0 is the slow one
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, times, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms, value in got:
        assert ms == max(times)          # every rank reports the slowest rank's time
        assert value == pytest.approx(world * bench.FLOPS / (max(times) / 1e3) / 1e12)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.5, None, torch.device("cpu")) == 3.5
    assert bench.whole_job_tflops(1, 1000.0) == pytest.approx(bench.FLOPS / 1e12)


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "3"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
