"""Host logic of a multi-GPU run, exercised with two gloo ranks on the CPU.

Every GPU runs an independent replica of the layer (no data-path collective),
so what a multi-rank run adds is host logic: per-rank seeds, the barrier
around the timed region, the maximum of the timings over ranks, the whole-job
throughput, the reference arm printing on rank 0 only, and failing (not
hanging) when a rank disappears."""
import datetime
import os
import socket
import sys
import time

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _init(rank, world, port, timeout_s=60):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=timeout_s))


def _worker_timing(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import bench
    from long_context_sequence_all_b200.workloads import WORKLOADS
    _init(rank, world, port)
    try:
        bench._barrier(world)
        ms = 10.0 + 5.0 * rank                        # rank 1 is the slow replica
        ms_max = bench._max_over_ranks(ms, world, torch.device("cpu"))
        seed = bench.rank_seed(WORKLOADS["qwen64k"], rank)
        q.put((rank, ms_max, seed, bench.job_throughput(65536, world, ms_max)))
        bench._barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_seeds_and_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker_timing, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, m0, s0, v0), (r1, m1, s1, v1) = res
    assert m0 == m1 == 15.0                           # max over ranks, the same everywhere
    assert s0 != s1                                   # each replica draws its own batch
    assert v0 == v1 == pytest.approx(2 * 65536 / 0.015)


def _worker_dies(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import bench
    _init(rank, world, port, timeout_s=5)
    if rank == 1:
        os._exit(3)                                   # this replica is gone before the barrier
    t0 = time.time()
    try:
        bench._barrier(world)
        q.put(("no error", time.time() - t0))
    except Exception as e:                            # the collective fails instead of hanging
        q.put((type(e).__name__, time.time() - t0))
    q.close()
    q.join_thread()                                   # flush the result before leaving
    os._exit(0)


def test_lost_rank_fails_the_barrier_instead_of_hanging():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker_dies, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    kind, waited = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
    assert kind != "no error"
    assert waited < 60


def test_reference_arm_runs_on_rank_zero_only():
    sys.path.insert(0, ROOT)
    import bench

    class A:
        workload, steps, warmup = "qwen64k", 1, 3
    assert bench.run_reference(A, rank=1, world=2) is None


def test_bench_gpus_flag_launches_one_rank_per_gpu():
    """`bench.py --gpus N` started directly runs the same command as N ranks
    (torch.distributed.run on 127.0.0.1); a WORLD_SIZE that disagrees with
    --gpus stops it with a message."""
    import subprocess
    sys.path.insert(0, ROOT)
    import bench
    cmd = bench.launch_command(4, ["--gpus", "4", "--steps", "2"])
    assert "torch.distributed.run" in cmd and "--nproc-per-node=4" in cmd
    assert cmd[cmd.index("--master-addr") + 1] == "127.0.0.1"
    assert cmd[-4:] == ["--gpus", "4", "--steps", "2"] and cmd[-5].endswith("bench.py")
    env = dict(os.environ, WORLD_SIZE="3", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2"], env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode != 0 and "WORLD_SIZE=3" in (r.stderr + r.stdout)
