"""Host-side multi-rank logic of the bench, as two gloo ranks on the CPU.

Decode over independent sequences shards by sequence with no exchange: each
rank decodes its own seeded batch, and the bench reduces only timings (max over
ranks) and byte counts (sum over ranks).  This checks those reductions and the
per-rank workloads over a real torch.distributed process group.
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
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime

    import torch
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    cpu = torch.device("cpu")
    mx = bench.max_over_ranks(1.5 * (rank + 1), world, cpu)
    sm = bench.sum_over_ranks(1000.0 + rank, world, cpu)
    w = bench.rank_workload("gqa", rank, world)
    bench.barrier(world)
    out.put((rank, mx, sm, w.seed, w.batch))
    dist.destroy_process_group()


def test_two_gloo_ranks_reduce_times_and_bytes():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, mx0, sm0, seed0, b0), (r1, mx1, sm1, seed1, b1) = res
    assert mx0 == mx1 == 3.0             # slowest rank decides the step time
    assert sm0 == sm1 == 2001.0          # bytes of all ranks are counted
    assert seed0 != seed1 and b0 == b1   # independent batches, same shapes


def test_single_rank_reductions_are_identity():
    sys.path.insert(0, ROOT)
    import torch

    import bench
    assert bench.max_over_ranks(2.5, 1, torch.device("cpu")) == 2.5
    assert bench.sum_over_ranks(7.0, 1, torch.device("cpu")) == 7.0
    assert bench.rank_workload("gqa", 0, 1).seed == 1002
