"""The multi-GPU bench path's host logic on CPU ranks (gloo, world size 2).

Decode and quantize-append partition by sequence with no exchange step, so
bench.py gives every rank its own batch and reduces only two things: the
timed region's length (max over ranks) and the work done (sum over ranks).
This runs that reduction on two CPU processes and checks the semantics.
"""

import os
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    times = [10.0 + rank, 20.0 - rank, 1.5 * (rank + 1)]
    counts = [1000.0 * (rank + 1), 7.0]
    t, c = bench.aggregate_across_ranks(times, counts, world, torch.device("cpu"))
    q.put((rank, t, c))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_reduction_max_time_sum_work():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, c in results:
        assert t == [11.0, 20.0, 3.0]          # max over ranks
        assert c == [3000.0, 14.0]             # sum over ranks


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    t, c = bench.aggregate_across_ranks([1.0, 2.0], [3.0], 1, torch.device("cpu"))
    assert t == [1.0, 2.0] and c == [3.0]
