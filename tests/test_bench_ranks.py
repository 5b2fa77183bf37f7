"""Multi-rank plumbing of bench.py on CPU (gloo, world size 2).

The decode path shards into independent replicas (every (request, head)
state is independent, no exchange step), so the only cross-rank work is the
timing aggregation: the whole-job value is all ranks' units over the slowest
rank's time.  This test runs that aggregation in two gloo processes.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, ws, port, out):
    import datetime
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    import bench
    units = 1000.0 * (rank + 1)
    secs = 0.5 + rank          # rank 1 is the slow one
    value, smax = bench.replica_throughput(units, secs, ws)
    bench.barrier(ws)
    out[rank] = (value, smax)
    dist.destroy_process_group()


def test_replica_throughput_two_ranks():
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
    assert out[0] == out[1] == (3000.0 / 1.5, 1.5)


def test_layer_range_partition():
    import bench
    for L in (1, 7, 20, 48):
        for ws in range(1, min(L, 9) + 1):
            ranges = [bench.layer_range(L, ws, r) for r in range(ws)]
            assert ranges[0][0] == 0 and ranges[-1][1] == L
            for (a, b), (c, d) in zip(ranges, ranges[1:]):
                assert b == c                      # contiguous, disjoint
            sizes = [b - a for a, b in ranges]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1
    with pytest.raises(ValueError):
        bench.layer_range(4, 5, 0)


def _shard_worker(rank, ws, port, out):
    import datetime
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    import bench
    lb, le = bench.layer_range(48, ws, rank)
    units = 70 * (le - lb) * 48 * 10           # head-steps of this rank's layers over 10 steps
    secs = 1.0 + 0.25 * rank
    value, smax = bench.replica_throughput(units, secs, ws)
    bench.barrier(ws)
    out[rank] = (value, smax)
    dist.destroy_process_group()


def test_layer_shards_cover_the_pool_once():
    # strong scaling: the ranks' layer shards add up to one whole pool step
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_shard_worker, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
    assert out[0] == out[1] == (70 * 48 * 48 * 10 / 1.25, 1.25)


def _prefill_worker(rank, ws, port, shard, out):
    import datetime
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    import bench
    L, H, n, T, steps = 48, 48, 1, 2048, 5
    lb, le = (0, L) if shard == "replicas" else bench.layer_range(L, ws, rank)
    secs = 2.0 + rank
    head_tokens, smax = bench.replica_throughput(n * T * steps * (le - lb) * H, secs, ws)
    bench.barrier(ws)
    out[rank] = (head_tokens / (L * H), smax)
    dist.destroy_process_group()


@pytest.mark.parametrize("shard,expect", [("layers", 2048 * 5 / 3.0), ("replicas", 2 * 2048 * 5 / 3.0)])
def test_prefill_tokens_per_second_two_ranks(shard, expect):
    # prefill counts tokens through the whole pool: layer shards split one pool's tokens,
    # replicas each prefill their own pool
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_prefill_worker, args=(2, port, shard, out), nprocs=2, join=True, start_method="spawn")
    assert out[0] == out[1]
    assert abs(out[0][0] - expect) < 1e-6 * expect and out[0][1] == 3.0
