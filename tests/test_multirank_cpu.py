"""The multi-rank path of bench.py on CPU: two gloo ranks (one process each,
rendezvous on 127.0.0.1) take the barrier and the max over ranks of the
step time exactly as the GPU ranks do over NCCL; the reference arm does its
work on rank 0 only; the whole-job value of N replicas is N times one
rank's work over the slowest rank's time."""
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


def _rank_main(rank, world, port, step_ms, out):
    import datetime

    import torch.distributed as dist

    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench._barrier(world)
        t = bench._allreduce_max(step_ms[rank], world, "cpu")
        bench._barrier(world)
        out.put((rank, t))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_step():
    world, port = 2, _free_port()
    step_ms = [1.25, 3.5]
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, step_ms, out)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict(out.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got == {0: 3.5, 1: 3.5}


def test_single_rank_needs_no_process_group():
    import bench
    assert bench._allreduce_max(2.5, 1, "cpu") == 2.5
    bench._barrier(1)  # no process group: returns at once


def test_job_value_is_weak_scaling_over_the_slowest_rank():
    import bench
    # one rank: 2e12 operations in 1 ms is 2000 TOPS
    assert bench._job_tops(2e12, 1.0, 1) == pytest.approx(2000.0)
    # four replicas each doing the same work, the slowest taking 2 ms
    assert bench._job_tops(2e12, 2.0, 4) == pytest.approx(4000.0)


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1", MASTER_ADDR="127.0.0.1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""
