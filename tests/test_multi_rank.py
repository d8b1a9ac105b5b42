"""Multi-rank host logic of the bench on CPU: two gloo ranks, no GPU.

The path shards by (batch, head) with no data exchange; a multi-GPU run is a
set of weak-scaled replicas whose only collectives are the timing reductions.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import datetime
    import sys
    import torch
    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    ms = [3.0, 5.0][rank]
    fl = [1e12, 2e12][rank]
    out = bench.aggregate_over_ranks(ms, fl, world, torch.device("cpu"))
    seeds = bench.rank_seed(1002, rank)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, out, seeds))


def test_weak_scaling_aggregation_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, (ms, fl), seed in res:
        assert ms == 5.0            # slowest rank
        assert fl == 3e12           # work of all ranks
    assert res[0][2] != res[1][2]   # each replica draws its own inputs


def test_single_rank_aggregation_is_identity():
    import bench
    assert bench.aggregate_over_ranks(4.0, 7.0, 1, None) == (4.0, 7.0)
