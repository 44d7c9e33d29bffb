"""The multi-rank plumbing of the benchmark on CPU (gloo, world size 2).

Heads (and batch elements) are independent attention problems, so ranks run
independent replicas with no collective on the data path; the only
cross-rank steps are the barrier around the timed region, the maximum of the
ranks' device times, and the whole-job aggregate (units of all ranks over
the slowest rank's time)."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    try:
        bench.barrier(world)
        m = bench.max_over_ranks(float(rank + 1) * 1.5, world)
        # weak scaling: every rank did the same units; the slowest time divides
        agg = bench.aggregate(100.0, 1.0 + rank, world)
        # head sharding: unequal units per rank are summed, the slowest time divides
        agg_sharded = bench.aggregate(10.0 * (rank + 1), 2.0, world)
        out.put((rank, m, agg, agg_sharded))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_and_aggregate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, m, agg, agg_sharded in res:
        assert m == 3.0                     # the max over ranks reaches every rank
        assert agg == pytest.approx(100.0 * 2 / 2.0)
        assert agg_sharded == pytest.approx((10.0 + 20.0) / 2.0)


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(2.5, 1) == 2.5
    assert bench.aggregate(10.0, 2.0, 1) == 5.0


@pytest.mark.parametrize("heads,world", [(40, 1), (40, 2), (40, 3), (40, 8), (24, 5), (7, 8)])
def test_shard_heads_partitions_the_heads(heads, world):
    """Head sharding (the path splits by head with no exchange step): the
    ranks' slices are contiguous, disjoint, cover every head and differ in
    size by at most one."""
    sys.path.insert(0, ROOT)
    from sparse_attention_video_tra_b200.runner import shard_heads
    seen = []
    sizes = []
    for r in range(world):
        first, count = shard_heads(heads, world, r)
        seen.extend(range(first, first + count))
        sizes.append(count)
    assert seen == list(range(heads))
    assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_heads(heads, world, world)
