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


def _plan_worker(rank, world, port, out):
    """--shard heads: each rank's workload slice and the plan it builds for it
    (host side only), gathered over the gloo group."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    from sparse_attention_video_tra_b200 import Plan
    try:
        args = bench.main.__globals__["argparse"].Namespace(
            workload="wan720", heads=0, retained=0.0, b=None, shard="heads", qsort="auto", gpus=world, calls=0)
        wl, total, (first, count) = bench.bench_workload(args, rank, world)
        p = Plan(wl.T, wl.H, wl.W, wl.heads, wl.d, wl.a, wl.b, wl.gamma, wl.Rt, wl.Bmin,
                 bench.query_group_flags("auto", wl))
        row = torch.tensor([first, count, p.info.heads, total], dtype=torch.int64)
        rows = [torch.zeros(4, dtype=torch.int64) for _ in range(world)]
        dist.all_gather(rows, row)
        out.put((rank, [r.tolist() for r in rows]))
        p.close()
    finally:
        dist.destroy_process_group()


def test_head_sharded_plans_partition_the_heads():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_plan_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = [q.get(timeout=10) for _ in range(2)]
    for _, rows in res:
        assert rows == res[0][1]                      # every rank sees the same table
        covered = []
        for first, count, plan_heads, total in rows:
            assert plan_heads == count > 0 and total == 40
            covered += list(range(first, first + count))
        assert sorted(covered) == list(range(40))     # disjoint and complete


def test_bench_gpus_2_starts_two_ranks():
    """`bench.py --gpus 2` outside torchrun starts 2 ranks itself (gloo here);
    the reference arm runs on rank 0 only and reports the head slices."""
    import json
    import subprocess
    env = dict(os.environ)
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT"):
        env.pop(k, None)
    p = subprocess.run([sys.executable, "bench.py", "--gpus", "2", "--impl", "reference", "--workload", "tiny",
                        "--shard", "heads", "--steps", "1", "--warmup", "0"], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stderr[-3000:]
    lines = [json.loads(x) for x in p.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1                            # rank 0 alone prints
    line = lines[0]
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["scaling"] == "strong"
    assert line["head_slices"] == [[0, 1], [1, 1]]
    assert line["config"]["global_batch"] == 2 and line["value"] > 0
