"""Host logic of the multi-process benchmark, on CPU with gloo (world size 2).

The op shards over (batch, head) with no exchange, so multi-GPU runs are
independent replicas; what needs checking is the host side: the timing
reduction takes the max over ranks, every rank takes the same collective
steps, and the reference arm does its work on rank 0 only.
"""
import multiprocessing as mp
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    t = bench.max_over_ranks(10.0 * (rank + 1), world)
    bench.barrier(world)

    class Args:
        steps, warmup, gpus = 1, 3, world
    rc = bench.run_reference(Args, world, rank) if rank != 0 else 0
    out.put((rank, t, rc))
    dist.destroy_process_group()


def test_max_over_ranks_and_reference_rank_rule():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(out.get(timeout=10) for _ in procs)
    # every rank sees the slowest rank's time; rank 1 returns from the
    # reference arm without doing any work
    assert res == [(0, 20.0, 0), (1, 20.0, 0)]


def test_workload_shape_override():
    sys.path.insert(0, ROOT)
    import bench

    class Args:
        shape = "2,4,1024,128"
    w = bench.workload_from_args(Args)
    assert (w.B, w.H, w.N, w.D) == (2, 4, 1024, 128)
    Args.shape = ""
    assert bench.workload_from_args(Args) is bench.WORKLOAD
