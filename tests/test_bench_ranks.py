"""The multi-rank path of bench.py on CPU: two gloo ranks (one process each)
agree on the slowest rank's step time and report whole-job throughput for
weak scaling (every rank compresses its own cache; no data-path collective)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(dist, 10.0 + 5.0 * rank, torch.device("cpu"))
        out[rank] = (ms, bench.weak_scaling_value(1e9, world, ms))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        mp.start_processes(_rank, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
        res = dict(out)
    assert res[0][0] == pytest.approx(15.0) and res[1][0] == pytest.approx(15.0)
    # 2 ranks x 1 GB in 15 ms
    assert res[0][1] == pytest.approx(2e9 / 15e-3 / 1e9)


def test_single_rank_needs_no_collective():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(None, 12.5, torch.device("cpu")) == 12.5
    assert bench.weak_scaling_value(2e9, 1, 1000.0) == pytest.approx(2.0)


def test_head_shards_partition_every_cache():
    """Strong scaling shares one cache by heads: the ranks' contiguous shares
    cover every head exactly once and differ in size by at most one."""
    import sys
    sys.path.insert(0, ROOT)
    import bench
    for H in (1, 7, 12, 32):
        for world in range(1, H + 1):
            shares = [bench.shard_units(H, world, r) for r in range(world)]
            assert shares[0][0] == 0 and shares[-1][1] == H
            assert all(shares[r][1] == shares[r + 1][0] for r in range(world - 1))
            sizes = [b - a for a, b in shares]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1
    # whole-job rate: the one cache's bytes over the slowest rank's time
    assert bench.strong_scaling_value(2e9, 1000.0) == 2.0


def test_share_blocks_cover_the_cache_once():
    """The ranks' block lists, in the cache's layer-major K-then-V order,
    partition every block of the cache exactly once."""
    from bit_kv_cache_qvg_b200.shard import share_blocks
    for L, H in ((1, 1), (3, 7), (2, 32)):
        for world in (1, 2, 3, min(H, 5)):
            parts = [share_blocks(L, H, world, r) for r in range(world)]
            flat = sorted(b for p in parts for b in p)
            assert flat == list(range(L * 2 * H))
            for p in parts:                       # each share keeps the cache's order
                assert p == sorted(p)
