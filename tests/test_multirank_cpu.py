"""The multi-rank path of bench.py on CPU: two gloo ranks (world size 2).

Units are independent, so each rank runs its own replica of the workload (weak
scaling, no collective on the data path); the only collective is the max of the
ranks' step times, taken in the same order by every rank.
"""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime
    import sys
    import torch
    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    from syngen import configs as C
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w = bench.rank_workload(C.get_workload("llama8b_32layers_b8_32k"), rank)
        my_ms = 1.0 + rank * 0.5                      # rank 1 is the slower one
        worst = bench.max_over_ranks(my_ms, world, torch.device("cpu"))
        e2e = bench.max_over_ranks(10.0 - rank, world, torch.device("cpu"))
        dist.barrier()
        q.put((rank, w.seed, worst, e2e, bench.aggregate_steps_per_s(worst, world)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_weak_scaling():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    seeds = [r[1] for r in res]
    assert len(set(seeds)) == world                 # each rank has its own units
    assert all(r[2] == 1.5 for r in res)            # max over ranks, seen by every rank
    assert all(r[3] == 10.0 for r in res)
    assert all(abs(r[4] - world * 1e3 / 1.5) < 1e-9 for r in res)   # whole-job steps/s


def test_single_rank_is_identity():
    import bench
    from syngen import configs as C
    w = C.get_workload("tiny")
    assert bench.rank_workload(w, 0) is w
    assert bench.max_over_ranks(3.25, 1, "cpu") == 3.25
    assert bench.aggregate_steps_per_s(2.0, 1) == 500.0
