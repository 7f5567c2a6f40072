"""Multi-rank host logic of the benchmark on CPU: world size 2 over gloo.

The operator shards with no exchange (every (b, c) chain is independent), so
N GPUs run N replicas; what must hold across ranks is the timing rule (the
slowest rank's time, reduced on every rank in the same collective order)
and the whole-job throughput (units of all ranks over that time).
"""
import os
import socket
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import datetime
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ws, r, local = bench.dist_env()
        assert (ws, r, local) == (world, rank, rank)
        # rank r pretends its timed region took 1 + r ms; every rank must see the max
        t = bench.max_over_ranks(1.0 + rank, dist, "cpu")
        t2 = bench.max_over_ranks(5.0 - rank, dist, "cpu")  # second collective, same order
        out[rank] = (t, t2, bench.aggregate_rate(1000, ws, t))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_aggregate_rate_gloo_world2():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world,
                       start_method="spawn", join=True)
    for r in range(world):
        t, t2, rate = out[r]
        assert t == 2.0 and t2 == 5.0
        assert rate == pytest.approx(2 * 1000 / 2.0e-3)


def test_single_rank_helpers_without_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, None, "cpu") == 3.5
    assert bench.aggregate_rate(10, 1, 1.0) == pytest.approx(1e4)
