"""The multi-GPU path is replicas only: every rank runs the whole decode batch, and the bench
takes the slowest rank's time and counts every rank's rows.  These tests run that host logic as
two gloo ranks on the CPU (no GPU, no NCCL)."""
import datetime
import os
import socket
import types

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, times, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        barrier, max_over_ranks = bench.rank_ops(dist, torch.device("cpu"))
        barrier()
        t = max_over_ranks(times[rank])
        barrier()
        q.put((rank, t, bench.replica_throughput(world, 64, 5, t)))
    finally:
        dist.destroy_process_group()


def test_two_ranks_agree_on_the_slowest_time_and_count_all_rows():
    world, port = 2, _free_port()
    times = [10.0, 12.5]                       # rank 1 is the slower replica
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, times, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, t, v in got:
        assert t == 12.5
        assert v == world * 64 * 5 / 12.5e-3


def test_single_process_needs_no_group():
    barrier, max_over_ranks = bench.rank_ops(None, torch.device("cpu"))
    barrier()
    assert max_over_ranks(3.25) == 3.25
    assert bench.replica_throughput(1, 64, 10, 2.0) == 64 * 10 / 2e-3


def test_reference_arm_runs_on_rank_zero_only(capsys):
    args = types.SimpleNamespace(gpus=2, steps=1, warmup=3)
    assert bench.run_reference(args, rank=1, world=2) is None
    assert capsys.readouterr().out == ""
