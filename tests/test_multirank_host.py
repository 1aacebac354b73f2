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


def _worker_distributed_ulysses(rank, world, port, results):
    """Ulysses over two real ranks (gloo): the exchange of the first and second
    all-to-alls, the attention layer and the loss aggregation of
    long_context_sequence_all_b200.distributed, with the oracle's routines as
    the pack / unpack / attention steps (the library runs its CUDA kernels
    there on GPUs)."""
    sys.path.insert(0, ROOT)
    import numpy as np
    import oracle
    from long_context_sequence_all_b200 import distributed as D
    _init(rank, world, port)
    try:
        rng = np.random.default_rng(11)
        B, n, H, G, d = 2, 24, 4, 2, 8
        s, hl, gl = n // world, H // world, G // world
        Q, K, V = (rng.standard_normal((B, n, h, d)) for h in (H, G, G))
        shard = lambda X: torch.from_numpy(np.ascontiguousarray(X[:, rank * s:(rank + 1) * s]))
        q, k, v = shard(Q), shard(K), shard(V)
        pack = lambda x: torch.from_numpy(oracle.seq_to_head(x.numpy()[None], x.shape[0], x.shape[1], 1,
                                                             x.shape[2])[0])
        unpack = lambda t: torch.from_numpy(oracle.head_to_seq(t.numpy()[None], t.shape[0], t.shape[2], 1,
                                                               t.shape[1])[0])
        # first all-to-all: this rank's slice of the oracle's logical-rank permutation
        qh = D.seq_to_head(q, pack=pack)
        seq_stack = lambda X: np.ascontiguousarray(X.reshape(B, world, s, X.shape[2], d).transpose(1, 0, 2, 3, 4))
        ref = oracle.seq_to_head(seq_stack(Q), B, n, world, H)[rank]
        ok_perm = bool(np.array_equal(qh.numpy(), ref))
        ok_back = bool(torch.equal(D.head_to_seq(qh, unpack=unpack), q))

        def attn(qh_, kh_, vh_, mask, cu, scale):
            nat = lambda t: np.ascontiguousarray(t.numpy().transpose(0, 2, 1, 3))      # [B][n][h][d]
            o, lse = oracle.attention_fwd(nat(qh_), nat(kh_), nat(vh_), mask=mask, cu_seqlens=cu, scale=scale)
            return torch.from_numpy(np.ascontiguousarray(o.transpose(0, 2, 1, 3))), torch.from_numpy(lse)

        O, _ = D.attention(q, k, v, mask=oracle.MASK_CAUSAL, attn=attn, pack=pack, unpack=unpack)
        O_full, _ = oracle.attention_fwd(Q.astype(np.float32), K.astype(np.float32), V.astype(np.float32),
                                         mask=oracle.MASK_CAUSAL)
        err = float(np.abs(O.numpy() - O_full[:, rank * s:(rank + 1) * s]).max())
        # the token-weighted loss: per-rank (S_r, C_r), one all-reduce
        T, Vv = 12, 16
        Z = rng.standard_normal((world * T, Vv)).astype(np.float32)
        Y = rng.integers(0, Vv, world * T).astype(np.int32)
        Y[::3] = -100
        Y[T:2 * T] = -100                               # rank 1's shard has no valid token
        S_r, C_r, _, _ = oracle.loss_aggregate(Z[rank * T:(rank + 1) * T], Y[rank * T:(rank + 1) * T], 1)
        L, C = D.aggregate_loss(float(S_r[0]), int(C_r[0]))
        _, _, L_ref, _ = oracle.loss_aggregate(Z, Y, world)
        results.put((rank, ok_perm, ok_back, err, abs(L - L_ref), C))
    finally:
        dist.destroy_process_group()


def test_two_rank_ulysses_exchange_layer_and_loss():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker_distributed_ulysses, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
    for rank, ok_perm, ok_back, err, lerr, C in res:
        assert ok_perm and ok_back, (rank, ok_perm, ok_back)
        assert err < 1e-6, (rank, err)           # float32 inputs, fp64 attention on both sides
        assert lerr < 1e-12 and C == res[0][5]
