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


def test_head_ranges_partition_the_heads():
    from block_sparse_attention_row_b200 import head_range
    for n in (0, 1, 5, 13, 40, 48, 97):
        for world in (1, 2, 3, 4, 8):
            got = [head_range(n, world, r) for r in range(world)]
            assert got[0][0] == 0 and got[-1][1] == n
            assert all(a[1] == b[0] for a, b in zip(got, got[1:]))          # contiguous, in rank order
            sizes = [hi - lo for lo, hi in got]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        head_range(4, 2, 2)


def _sharded_worker(rank, world, port, q):
    import datetime
    import sys
    import numpy as np
    import torch
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import oracle as O
    from block_sparse_attention_row_b200 import head_range, head_shard
    from synth import make_qkv_custom
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    B, H, N, d, bq, bk, k, p = 2, 3, 300, 16, 64, 64, 0.2, 0.8
    # Every rank holds the same layer (same seed) and takes its own heads of it.
    Q, K, V = make_qkv_custom(B, H, N, d, seed=7, positional_field=True, sink_heads=(0,), uniform_heads=(1,))
    Qs, Ks, Vs = (head_shard(x, world, rank) for x in (Q, K, V))
    _, cnt, idx, _ = O.hybrid_mask(Qs, Ks, bq, bk, k, p)
    Os, _ = O.block_sparse_attention(Qs, Ks, Vs, cnt, idx, bq, bk)
    parts = [None] * world
    dist.all_gather_object(parts, (head_range(B * H, world, rank), cnt, idx, Os))
    dist.barrier()
    dist.destroy_process_group()
    if rank == 0:
        _, cnt_w, idx_w, _ = O.hybrid_mask(Q, K, bq, bk, k, p)
        O_w, _ = O.block_sparse_attention(Q, K, V, cnt_w, idx_w, bq, bk)
        flat = lambda a: a.reshape((B * H,) + a.shape[2:])
        ok = True
        covered = []
        for (lo, hi), c, i, o in parts:
            covered += list(range(lo, hi))
            ok &= np.array_equal(c[0], flat(cnt_w)[lo:hi]) and np.array_equal(i[0], flat(idx_w)[lo:hi])
            ok &= np.array_equal(o[0], flat(O_w)[lo:hi])
        q.put((ok, covered))
    else:
        q.put(None)


def test_head_sharded_layer_equals_the_whole_layer_two_gloo_ranks():
    """Two ranks each run the path (the oracle, on CPU) on their heads of one
    layer; gathered, the shards equal the whole layer's lists and output."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_sharded_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    ok, covered = next(r for r in res if r is not None)
    assert covered == list(range(6))
    assert ok


def test_head_shard_is_a_contiguous_view_of_the_layer():
    import torch
    from block_sparse_attention_row_b200 import head_range, head_shard
    X = torch.arange(2 * 5 * 3 * 4, dtype=torch.float32).reshape(2, 5, 3, 4)
    flat = X.reshape(10, 3, 4)
    for world in (1, 3, 4):
        for r in range(world):
            lo, hi = head_range(10, world, r)
            S = head_shard(X, world, r)
            assert S.shape == (1, hi - lo, 3, 4) and S.is_contiguous()
            assert S.data_ptr() == flat[lo:].data_ptr() if hi > lo else True
            assert torch.equal(S[0], flat[lo:hi])
    with pytest.raises(ValueError):
        head_shard(X.transpose(1, 2), 2, 0)
