"""Benchmark of the Token Radius Attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload wan720] [--impl tra|reference]

With --gpus N > 1 and no torchrun environment, the script starts N ranks of
itself through torch.distributed.run on this node (one per GPU); under
torchrun it checks that WORLD_SIZE equals N.

A step is one pass of the whole hot path over one batch of synthetic input:
dense (or key-subsampled) warm-up entropy, one radius/mask build, then
`calls` attention calls that reuse the mask with a fresh V each (10 for the
Wan-14B-720p shape: 21x45x80 tokens, 40 heads, d=128, bf16).  The headline
value is the retained-pair throughput of the attention calls: 4*d FLOPs per
retained token pair (the pairs the radius mask keeps, not the padded tiles
the kernel computes) over their device time, summed over ranks (heads are
independent, so ranks run independent replicas: weak scaling, no collective
on the data path).  Inputs are resident in HBM and larger than L2; L2 is
also flushed before every step.

`--impl reference` runs the fp64 CPU oracle (the only reference this method
has) on a bounded sample of the same workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
# B200 exponential unit (MUFU ex2): 16 results per clock per SM, 148 SMs, at
# the 1965 MHz maximum SM clock -- the bound of the entropy kernel
MUFU_EX2_PER_S = 16 * 148 * 1965e6
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
METRIC = "TRA attention retained-pair TFLOP/s (bf16) at 21x45x80 tokens, 40 heads; ms/call reported"


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def peak_value(key: str):
    """One roofline denominator: (value, "measured"|"fallback").  The measured
    file's number when it holds one under `key`, else the profiling recipe's
    fallback, labelled as such."""
    pk, kind = peaks()
    v = pk.get(key) if isinstance(pk, dict) else None
    if kind == "measured" and isinstance(v, (int, float)) and not isinstance(v, bool) and v > 0:
        return float(v), "measured"
    return float(FALLBACK_PEAKS[key]), "fallback"


# ---------------------------------------------------------------- distributed
def dist_setup(expected_world: int = 0):
    """Rank and world size from the torchrun environment; one process per GPU
    (LOCAL_RANK picks the device).  NCCL when GPUs are present, else gloo
    (the CPU tests).  The process group gets a short timeout so that ranks
    waiting on a rank that died end with an error instead of hanging."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if expected_world and world != expected_world:
        raise SystemExit(f"bench.py: --gpus {expected_world} but WORLD_SIZE={world}")
    if torch.cuda.is_available():
        if local >= torch.cuda.device_count():
            raise SystemExit(f"bench.py: LOCAL_RANK {local} but only {torch.cuda.device_count()} GPUs are visible")
        torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=180))
    return rank, world


def relaunch(argv, n: int) -> int:
    """Start n ranks of this script on this node through torch.distributed.run
    (rendezvous on 127.0.0.1, a free port); returns their exit status."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", f"--master-port={port}", os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def sum_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def aggregate(per_rank_units: float, per_rank_seconds: float, world: int) -> float:
    """Whole-job throughput: units of all ranks over the slowest rank's time."""
    return sum_over_ranks(per_rank_units, world) / max_over_ranks(per_rank_seconds, world)


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clock/throttle samples during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.path = os.path.join("/tmp", f"tra_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- profiles
ROOFLINE_KERNEL = "attention_kernel"     # the dominant kernel; its ncu summary is profiles/<kernel>_<workload>_*


def source_sha256() -> str:
    """sha256 over every file of the kernel source directory, in name order."""
    from sparse_attention_video_tra_b200.build import CSRC
    import hashlib
    h = hashlib.sha256()
    for f in sorted(os.listdir(CSRC)):
        h.update(open(os.path.join(CSRC, f), "rb").read())
    return h.hexdigest()


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", f"{kernel}_{workload}_traffic.txt")
    if not os.path.exists(p):
        return None
    kv = {}
    for line in open(p):
        if ":" in line and not line.startswith("#"):
            k, v = line.split(":", 1)
            kv[k.strip()] = v.strip()
    if kv.get("source_sha256") != source_sha256():
        return None
    try:
        return float(kv["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# ---------------------------------------------------------------- oracle (CPU)
def oracle_sample(wl, b, budget_s: float, rng_seed: int, heads=(0,), device="cuda", metric: int = 0):
    """Time the fp64 oracle's whole path (entropy, radius, attention) on a
    bounded random sample of queries of the same workload.  Returns the
    retained-pair TFLOP/s it reached and a description."""
    sys.path.insert(0, ROOT)
    import oracle
    from sparse_attention_video_tra_b200 import synth
    T, H, W, d = wl.T, wl.H, wl.W, wl.d
    N = wl.N
    q, k, v = synth.make_qkv(T, H, W, wl.heads, d, synth.SEED_BASE + wl.index, device=device,
                             dtype=torch.bfloat16)
    sel = list(heads)

    def bits(x):
        return x[sel].cpu().contiguous().view(torch.int16).numpy().view(np.uint16)

    qb, kb, vb = bits(q), bits(k), bits(v)
    del q, k, v
    G = len(sel)
    rng = np.random.default_rng(rng_seed)
    threads = oracle.num_threads()

    def run(nq):
        idx = np.sort(rng.choice(G * N, size=nq, replace=False))
        t0 = time.perf_counter()
        Hs = oracle.entropy(qb, kb, G, (T, H, W), d, key_stride=wl.key_stride, ktile=(8, 16), queries=idx) \
            if wl.key_stride == 1 else _oracle_entropy_tiled(oracle, qb, kb, G, wl, idx)
        r, c, _ = oracle.radius(Hs.astype(np.float32), G, (T, H, W), wl.a, b, wl.gamma, wl.Rt, wl.Bmin, queries=idx,
                                metric=metric)
        r_all = np.zeros(G * N, np.int32)
        r_all[idx] = r
        oracle.attention(qb, kb, vb, r_all, G, (T, H, W), d, wl.gamma, wl.Rt, queries=idx, metric=metric)
        dt = time.perf_counter() - t0
        return dt, int(c.sum()), nq

    nq = max(threads, 4)
    dt, pairs, nq = run(nq)
    while dt < budget_s / 3 and nq < G * N:
        nq = int(min(G * N, nq * min(8.0, max(2.0, budget_s / max(dt, 1e-3)))))
        dt, pairs, nq = run(nq)
    tflops = 4.0 * d * pairs / dt / 1e12
    return tflops, {"queries": nq, "heads": sel, "seconds": round(dt, 3), "threads": threads,
                    "retained_pairs": pairs}


def oracle_parity(run, wl, n_queries: int = 256, seed: int = 77):
    """Part of the CPU-baseline leg: the fp64 oracle on a random sample of head
    0's queries against this run's GPU results at full size -- entropy
    (relative error), radii from the GPU's entropies (mismatches; bit-exact
    expected) and attention rows of call 0 with those radii (max/mean abs)."""
    sys.path.insert(0, ROOT)
    import oracle
    T, H, W, d, N = wl.T, wl.H, wl.W, wl.d, wl.N
    i = run.info
    run.run_attention(0)
    torch.cuda.synchronize()
    # tile-major row -> natural token for head 0
    p = np.arange(i.N_pad)
    tile, inn = p // 128, p % 128
    tpf = i.n_tiles_h * i.n_tiles_w
    t, rem = tile // tpf, tile % tpf
    hh = (rem // i.n_tiles_w) * i.tile_h + inn // i.tile_w
    ww = (rem % i.n_tiles_w) * i.tile_w + inn % i.tile_w
    valid = (hh < H) & (ww < W)
    nat = np.where(valid, (t * H + hh) * W + ww, -1)
    rows = np.sort(np.random.default_rng(seed).choice(np.nonzero(valid)[0], n_queries, replace=False))
    queries = nat[rows]
    order = np.argsort(queries)
    rows, queries = rows[order], queries[order]

    # natural-order head-0 inputs (bf16 bit patterns)
    from sparse_attention_video_tra_b200 import Plan
    p1 = Plan(T, H, W, 1, d, wl.a, run.b, wl.gamma, wl.Rt, wl.Bmin, run.plan.flags)
    nq = torch.empty((1, N, d), dtype=torch.bfloat16, device="cuda")
    bits = []
    for x in (run.q, run.k, run.v[0]):
        p1.permute(x[:1].contiguous(), nq, False)
        bits.append(nq.cpu().view(torch.int16).numpy().view(np.uint16).copy())
    p1.close()
    qb, kb, vb = bits
    Hg = run.H[0].cpu().numpy()[rows]
    if wl.key_stride == 1:
        Hr = oracle.entropy(qb, kb, 1, (T, H, W), d, queries=queries)
    else:
        Hr = _oracle_entropy_tiled(oracle, qb, kb, 1, wl, queries)
    from sparse_attention_video_tra_b200 import TRA_FLAG_DISK
    metric = oracle.DISK if run.plan.flags & TRA_FLAG_DISK else oracle.CHEBYSHEV
    rad = run.plan.mask_views(run.mask)[0][0].cpu().numpy()
    r_ref, _, _ = oracle.radius(Hg, 1, (T, H, W), wl.a, run.b, wl.gamma, wl.Rt, wl.Bmin, queries=queries,
                                metric=metric)
    r_all = np.zeros(N, np.int32)
    r_all[nat[valid]] = rad[valid]
    O = oracle.attention(qb, kb, vb, r_all, 1, (T, H, W), d, wl.gamma, wl.Rt, queries=queries, metric=metric)
    Og = run.out[0].float().cpu().numpy()[rows]
    err = np.abs(Og - O)
    return {"queries": int(n_queries), "head": 0,
            "entropy_max_rel": float(np.max(np.abs(Hg - Hr) / np.maximum(np.abs(Hr), 1.0))),
            "radius_mismatches": int(np.sum(rad[rows] != r_ref)),
            "attention_max_abs": float(err.max()), "attention_mean_abs": float(err.mean()),
            "tolerances": {"entropy_rel": 1e-3, "radius": "bit-exact", "attention_max_abs": 1e-2,
                           "attention_mean_abs": 1e-3}}


def _oracle_entropy_tiled(oracle, qb, kb, G, wl, idx):
    # key subsampling is defined on the library's key tiles: pass the plan's tile shape
    from sparse_attention_video_tra_b200 import Plan
    p = Plan(wl.T, wl.H, wl.W, 1, wl.d, 1.0, 0.0, wl.gamma, wl.Rt, wl.Bmin)
    th, tw = p.info.tile_h, p.info.tile_w
    p.close()
    return oracle.entropy(qb, kb, G, (wl.T, wl.H, wl.W), wl.d, key_stride=wl.key_stride, ktile=(th, tw), queries=idx)


# ---------------------------------------------------------------- workload and config (both arms)
def bench_workload(args, rank: int, world: int):
    """The workload this rank runs: the named one, with the command line's
    head count, retained fraction or b; with --shard heads only this rank's
    contiguous slice of the heads.  Returns (workload, all heads, the rank's
    (first head, count)).  Host-side only (no GPU)."""
    import dataclasses
    sys.path.insert(0, ROOT)
    from sparse_attention_video_tra_b200 import synth
    from sparse_attention_video_tra_b200.runner import shard_heads
    wl = synth.WORKLOADS[args.workload]
    if args.heads:
        wl = dataclasses.replace(wl, heads=args.heads, name=wl.name.replace(f"{wl.heads} heads", f"{args.heads} heads"))
    if args.retained:
        wl = dataclasses.replace(wl, target_retained=float(args.retained), b=None)
    if args.b is not None:
        wl = dataclasses.replace(wl, b=float(args.b))
    total = wl.heads
    first, count = 0, wl.heads
    if args.shard == "heads":
        first, count = shard_heads(wl.heads, world, rank)
        if count == 0:
            raise SystemExit(f"rank {rank}: no heads left to shard ({wl.heads} heads over {world} ranks)")
        wl = dataclasses.replace(wl, heads=count)
    return wl, total, (first, count)


def attention_calls(args) -> int:
    return args.calls if args.calls else (10 if args.workload == "wan720" else 1)


def bench_config(args, wl, total_heads: int, world: int, b: float) -> dict:
    """The `config` object of the JSON line, the same for both arms: the
    workload, the batch, the plan's parameters and tile choice."""
    from sparse_attention_video_tra_b200 import Plan, TRA_FLAG_QSORT
    sharded = args.shard == "heads"
    flags = plan_flags(args, wl)
    p = Plan(wl.T, wl.H, wl.W, 1, wl.d, wl.a, b, wl.gamma, wl.Rt, wl.Bmin, flags)
    tile_desc = f"1x{p.info.tile_h}x{p.info.tile_w}"
    p.close()
    return {"workload": args.workload_name if hasattr(args, "workload_name") else wl.name,
            "global_batch": total_heads if sharded else total_heads * max(world, 1), "seq_len": wl.N,
            "parallelism": (f"heads sharded over {world} GPUs, no collective on the path" if sharded
                            else f"independent head-batch replicas x{world}"),
            "attention_calls_per_step": attention_calls(args),
            "a": wl.a, "b": round(float(b), 6), "gamma": wl.gamma, "Rt": wl.Rt, "Bmin": wl.Bmin,
            "tile": tile_desc,
            "query_groups": "radius-sorted groups (TRA_FLAG_QSORT)" if flags & TRA_FLAG_QSORT else "spatial tiles",
            "metric": "Euclidean disk (TRA_FLAG_DISK)" if args.metric == "disk" else "Chebyshev square",
            "inputs": "resident in HBM, larger than L2; L2 flushed before every step"}


# ---------------------------------------------------------------- arms
def run_reference(args, rank, world):
    if rank != 0:
        return 0
    sys.path.insert(0, ROOT)
    import oracle
    wl, total_heads, _ = bench_workload(args, 0, 1)
    args.workload_name = synth_name(args, total_heads)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    # b: the workload's fixed value (the one the GPU arm uses); only a
    # target-fraction run finds its own, with the oracle on a query sample
    b = wl.b
    if b is None:
        b = _oracle_calibrate_b(oracle, wl, dev, oracle_metric(args))
    vals = []
    budget = max(2.0, min(20.0, 150.0 / max(1, args.steps + args.warmup)))
    for s in range(args.warmup + args.steps):
        v, desc = oracle_sample(wl, b, budget, 1234 + s, device=dev, metric=oracle_metric(args))
        if s >= args.warmup:
            vals.append((v, desc))
    value = float(np.mean([v for v, _ in vals]))
    desc = vals[-1][1]
    config = bench_config(args, wl, total_heads, world, b)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True,
            "scaling": "strong" if args.shard == "heads" else "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config,
            "sample": "random queries of head 0, whole oracle path (entropy, radius, attention)",
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": desc["threads"], "kind": "oracle",
                             "sample": f"{desc['queries']} queries of head 0 per step, entropy+radius+attention"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    if args.shard == "heads":
        from sparse_attention_video_tra_b200.runner import shard_heads
        line["head_slices"] = [list(shard_heads(total_heads, world, r)) for r in range(world)]
    print(json.dumps(line), flush=True)
    return 0


def synth_name(args, total_heads: int) -> str:
    from sparse_attention_video_tra_b200 import synth
    wl = synth.WORKLOADS[args.workload]
    return wl.name.replace(f"{wl.heads} heads", f"{total_heads} heads")


def _oracle_calibrate_b(oracle, wl, dev, metric: int = 0):
    from sparse_attention_video_tra_b200 import synth
    q, k, _ = synth.make_qkv(wl.T, wl.H, wl.W, wl.heads, wl.d, synth.SEED_BASE + wl.index, device=dev,
                             dtype=torch.bfloat16)
    qb = q[:1].cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    kb = k[:1].cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    del q, k
    rng = np.random.default_rng(99)
    idx = np.sort(rng.choice(wl.N, size=256, replace=False))
    if wl.key_stride == 1:
        Hs = oracle.entropy(qb, kb, 1, wl.grid, wl.d, queries=idx)
    else:
        Hs = _oracle_entropy_tiled(oracle, qb, kb, 1, wl, idx)
    lo, hi = -30.0, 30.0
    for _ in range(30):
        mid = 0.5 * (lo + hi)
        _, c, _ = oracle.radius(Hs.astype(np.float32), 1, wl.grid, wl.a, mid, wl.gamma, wl.Rt, wl.Bmin, queries=idx,
                                metric=metric)
        if c.mean() / wl.N < wl.target_retained:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def query_group_flags(mode: str, wl) -> int:
    """TRA_FLAG_QSORT when asked for, or (auto) when the plan accepts it and a
    frame has more than one tile row, so that a tile-column strip holds
    several tiles whose queries can be regrouped by radius (with one tile row
    the groups are the tiles themselves)."""
    from sparse_attention_video_tra_b200 import Plan, TRA_FLAG_QSORT, TraError
    if mode == "off":
        return 0
    try:
        p = Plan(wl.T, wl.H, wl.W, 1, wl.d, wl.a, 0.0, wl.gamma, wl.Rt, wl.Bmin, TRA_FLAG_QSORT)
        rows = p.info.n_tiles_h
        p.close()
    except TraError:
        if mode == "on":
            raise
        return 0
    return TRA_FLAG_QSORT if (mode == "on" or rows > 1) else 0


def plan_flags(args, wl) -> int:
    """The plan flags of a run: query groups (above) and the spatial test."""
    from sparse_attention_video_tra_b200 import TRA_FLAG_DISK
    return query_group_flags(args.qsort, wl) | (TRA_FLAG_DISK if args.metric == "disk" else 0)


def oracle_metric(args) -> int:
    sys.path.insert(0, ROOT)
    import oracle
    return oracle.DISK if args.metric == "disk" else oracle.CHEBYSHEV


def run_tra(args, rank, world):
    sys.path.insert(0, ROOT)
    from sparse_attention_video_tra_b200.runner import WorkloadRun
    # strong scaling (--shard heads): this rank's contiguous slice of the heads
    wl, total_heads, _ = bench_workload(args, rank, world)
    args.workload_name = synth_name(args, total_heads)
    calls = attention_calls(args)
    flags = plan_flags(args, wl)
    run = WorkloadRun(wl, calls=calls, seed_offset=rank, flags=flags)
    dev_idx = torch.cuda.current_device()
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device="cuda")
    nev = 3 + calls

    def timed_steps(k, record):
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)] for _ in range(k)]
        for s in range(k):
            flush.zero_()
            run.step(evs[s] if record else None, stream=None)
        return evs

    for _ in range(args.warmup):
        timed_steps(1, False)
    torch.cuda.synchronize()
    barrier(world)
    clocks = ClockSampler(dev_idx)
    clocks.start()
    torch.cuda.synchronize()
    barrier(world)
    t_wall0 = time.perf_counter()
    evs = timed_steps(args.steps, True)
    torch.cuda.synchronize()
    t_wall = time.perf_counter() - t_wall0
    barrier(world)
    clk = clocks.stop()

    step_ms = [e[0].elapsed_time(e[-1]) for e in evs]
    ent_ms = [e[0].elapsed_time(e[1]) for e in evs]
    mask_ms = [e[1].elapsed_time(e[2]) for e in evs]
    call_ms = [e[2 + c].elapsed_time(e[3 + c]) for e in evs for c in range(calls)]
    attn_s = sum(call_ms) / 1000.0
    flops = run.attention_flops()
    # value: all timed calls over their summed device time (the whole-job
    # rate); the per-phase figures below are medians over steps / calls
    value = aggregate(flops * calls * args.steps, attn_s, world) / 1e12
    step_s = sum(step_ms) / 1000.0
    step_tflops = aggregate(flops * calls * args.steps, step_s, world) / 1e12
    ms_per_step = max_over_ranks(float(np.median(step_ms)), world)

    # separate L2-flushed timing of the mask build (its inputs fit in L2)
    mask_runs = []
    for _ in range(5):
        flush.zero_()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record()
        run.run_mask()
        a1.record()
        torch.cuda.synchronize()
        mask_runs.append(a0.elapsed_time(a1))
    mask_cold_ms = float(np.median(mask_runs))

    avg_call_s = float(np.median(call_ms)) / 1000.0
    achieved = flops / avg_call_s / 1e12
    peak, pk_kind = peak_value("bf16_tflops_sustained")
    computed = run.computed_pairs()
    traffic = recorded_traffic(ROOFLINE_KERNEL, args.workload)
    roofline = {"bound": "tensor", "kernel": "tra::" + ROOFLINE_KERNEL, "achieved": round(achieved, 2),
                "peak": peak, "peak_kind": f"{pk_kind} bf16 sustained", "unit": "TFLOP/s",
                "frac": round(achieved / peak, 4), "traffic": traffic,
                "computed_tile_tflops": round(4.0 * wl.d * computed / avg_call_s / 1e12, 2),
                "computed_tile_frac": round(4.0 * wl.d * computed / avg_call_s / 1e12 / peak, 4),
                "tile_efficiency": round(run.retained_pairs / computed, 4),
                "frac_of_burst": round(achieved / peak_value("bf16_tflops")[0], 4)}
    mask_bytes_alg = mask_algorithmic_bytes(run)
    hbm, hbm_kind = peak_value("hbm_gbs")
    ent_s = float(np.median(ent_ms)) / 1000.0
    ent_rate = run.entropy_pairs() / ent_s
    ent_bytes = entropy_algorithmic_bytes(run)
    phases = {"statistic": "median over steps (attention: over calls)",
              "entropy_ms": round(ent_s * 1000.0, 3), "mask_ms": round(float(np.median(mask_ms)), 4),
              "mask_ms_l2_flushed": round(mask_cold_ms, 4),
              "mask_gbs": round(mask_bytes_alg / (mask_cold_ms / 1000.0) / 1e9, 2),
              "mask_hbm_frac": round(mask_bytes_alg / (mask_cold_ms / 1000.0) / 1e9 / hbm, 4),
              "hbm_peak": {"gbs": hbm, "kind": hbm_kind},
              "attention_ms_per_call": round(avg_call_s * 1000.0, 3),
              "entropy_scores_per_s": ent_rate,
              "entropy_roofline": {"bound": "alu", "unit": "exponentials/s", "achieved": ent_rate,
                                   "peak": MUFU_EX2_PER_S, "frac": round(ent_rate / MUFU_EX2_PER_S, 4),
                                   "peak_derivation": "one ex2 per scored pair; MUFU 16/clk/SM x 148 SMs x 1965 MHz",
                                   # the same bound at the median SM clock sampled over the
                                   # timed region (entropy is about a sixth of it; the long
                                   # kernels run at the power cap, below the 1965 MHz maximum)
                                   "frac_at_sampled_clock": (round(ent_rate / (16 * 148 * clk["sm_mhz"] * 1e6), 4)
                                                             if clk and clk.get("sm_mhz") else None),
                                   "dram_gbs": round(ent_bytes / ent_s / 1e9, 2),
                                   "dram_frac": round(ent_bytes / ent_s / 1e9 / hbm, 5),
                                   "algorithmic_bytes": ent_bytes}}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        v, desc = oracle_sample(wl, run.b, args.cpu_budget, 4321, metric=oracle_metric(args))
        cpu = {"value": v, "unit": "TFLOP/s", "cores": desc["threads"], "kind": "oracle",
               "sample": f"{desc['queries']} random queries of head 0: entropy+radius+attention in fp64, "
                         f"{desc['seconds']} s",
               "parity": oracle_parity(run, wl)}

    e2e = None if args.no_e2e else run_e2e(run, wl, calls, args, world)
    b_used, retained = run.b, run.retained_fraction_now()
    del run
    sharded = args.shard == "heads"
    line = {"metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 3),
            "higher_is_better": True, "scaling": "strong" if sharded else "weak", "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic (seeded Q,K,V with the video-DiT attention shapes; no model weights)",
            "config": bench_config(args, wl, total_heads, world, b_used),
            "retained_fraction": round(retained, 5), "phases": phases, "step_tflops": round(step_tflops, 3),
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": (2 + calls) * args.steps, "clocks": clk, "wall_s_timed": round(t_wall, 3)}
    return line


def entropy_algorithmic_bytes(run) -> float:
    """Bytes the entropy pass must move: Q and K once (bf16, the plan's rows)
    and one fp32 entropy per row."""
    i = run.info
    return i.heads * i.N_pad * (2.0 * i.d * 2 + 4.0)


def mask_algorithmic_bytes(run) -> float:
    """Bytes the mask build must move: read H (4 B/row), write r (4 B/row),
    per tile count (4 B) and pair sum (8 B), 2 B per listed key tile."""
    i = run.info
    listed = int(run.plan.mask_views(run.mask)[1].sum().item())
    groups = i.heads * i.N_pad * 1.0 if run.plan.qsort else 0.0      # 1 B per group slot
    return i.heads * i.N_pad * 8.0 + i.heads * i.n_tiles * 12.0 + 2.0 * listed + groups


def run_e2e(run, wl, calls, args, world):
    """The same metric through the public API with host buffers.  Per step:
    pinned host -> device copies of Q, K (natural token order) and of each
    call's V, the hot path on natural-layout plans (TRA_FLAG_NATURAL: the
    kernels read frame-major tensors through 4-D TMA boxes, no permute pass),
    and each call's output back to pinned host memory.

    Copies run on their own streams and overlap compute, within a step and
    across steps: Q and K are double-buffered by step, so the next step's
    upload runs during this step's last attention calls; V and the outputs are
    double-buffered by call, so V of call c+1 goes up while call c runs and
    each output comes down while later work runs.  The fences (an event per
    buffer) carry over from one step to the next; the timed region ends when
    the last output has landed in host memory.

    Heads are independent problems, so they may be split into chunks
    (--e2e-chunks), each with its own plan and mask buffer; with the
    cross-step overlap one chunk (one launch per call, no extra wave tails)
    is the default."""
    from sparse_attention_video_tra_b200 import Plan, TRA_FLAG_NATURAL
    from sparse_attention_video_tra_b200.runner import shard_heads
    i = run.info
    n_chunks = max(1, min(args.e2e_chunks, wl.heads))
    chunks = [shard_heads(wl.heads, n_chunks, c) for c in range(n_chunks)]
    plans = [Plan(wl.T, wl.H, wl.W, cnt, wl.d, wl.a, run.b, wl.gamma, wl.Rt, wl.Bmin,
                  run.plan.flags | TRA_FLAG_NATURAL) for _, cnt in chunks]
    shape = (i.heads, i.N, i.d)
    hq = torch.empty(shape, dtype=torch.bfloat16, pin_memory=True)
    hk = torch.empty(shape, dtype=torch.bfloat16, pin_memory=True)
    hv = torch.empty(shape, dtype=torch.bfloat16, pin_memory=True)
    ho = torch.empty(shape, dtype=plans[0].out_dtype, pin_memory=True)
    tmp = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    run.plan.permute(run.q, tmp, False); hq.copy_(tmp)
    run.plan.permute(run.k, tmp, False); hk.copy_(tmp)
    run.plan.permute(run.v[0], tmp, False); hv.copy_(tmp)
    del tmp
    dq = [torch.empty(shape, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    dk = [torch.empty_like(dq[0]) for _ in range(2)]
    dv = [torch.empty_like(dq[0]) for _ in range(2)]
    do = [torch.empty(shape, dtype=plans[0].out_dtype, device="cuda") for _ in range(2)]
    dH = torch.empty((i.heads, i.N), dtype=torch.float32, device="cuda")
    dmask = [p.new_mask() for p in plans]
    sl = [slice(g0, g0 + cnt) for g0, cnt in chunks]
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()                       # noqa: E731
    # fences carried across steps (None: the buffer is free)
    st = {"qk_free": [None, None], "v_free": [None, None], "o_free": [[None] * n_chunks for _ in range(2)],
          "last": None, "n": 0}

    def step():
        p = st["n"] & 1
        st["n"] += 1
        if st["qk_free"][p] is not None:                   # the step two back no longer reads set p
            s_in.wait_event(st["qk_free"][p])
        qk_in = []
        with torch.cuda.stream(s_in):
            for h in sl:
                dq[p][h].copy_(hq[h], non_blocking=True)
                dk[p][h].copy_(hk[h], non_blocking=True)
                qk_in.append(ev()); qk_in[-1].record(s_in)
        for pl, h, m, e in zip(plans, sl, dmask, qk_in):
            comp.wait_event(e)
            pl.entropy(dq[p][h], dk[p][h], dH[h], wl.key_stride, stream=comp)
            pl.radius_and_mask(dH[h], m, stream=comp)
        done = None
        for c in range(calls):
            b = c & 1
            if st["v_free"][b] is not None:
                s_in.wait_event(st["v_free"][b])
            with torch.cuda.stream(s_in):
                dv[b].copy_(hv, non_blocking=True)
                v_in = ev(); v_in.record(s_in)
            comp.wait_event(v_in)
            for q, (pl, h, m) in enumerate(zip(plans, sl, dmask)):
                if st["o_free"][b][q] is not None:
                    comp.wait_event(st["o_free"][b][q])
                pl.attention(dq[p][h], dk[p][h], dv[b][h], m, do[b][h], stream=comp)
                done = ev(); done.record(comp)
                s_out.wait_event(done)
                with torch.cuda.stream(s_out):
                    ho[h].copy_(do[b][h], non_blocking=True)
                    out_done = ev(); out_done.record(s_out)
                st["o_free"][b][q] = out_done
                st["last"] = out_done
            st["v_free"][b] = done
        st["qk_free"][p] = done

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    for _ in range(args.steps):
        step()
    comp.wait_event(st["last"])                            # every output in host memory
    e1.record(comp)
    torch.cuda.synchronize()
    barrier(world)
    if any(p.status() != 0 for p in plans):
        raise RuntimeError("device error word set during the end-to-end run")
    secs = e0.elapsed_time(e1) / 1000.0
    val = aggregate(run.attention_flops() * calls * args.steps, secs, world) / 1e12
    nbytes = i.heads * i.N * i.d * 2
    obytes = i.heads * i.N * i.d * ho.element_size()
    for p in plans:
        p.close()
    return {"value": round(val, 3), "unit": "TFLOP/s", "h2d_bytes_per_step": nbytes * (2 + calls),
            "d2h_bytes_per_step": obytes * calls, "ms_per_step": round(secs * 1000.0 / args.steps, 3),
            "head_chunks": n_chunks,
            "layout": "natural [heads][T][H][W][d]; copies on two copy streams, overlapped with compute "
                      "within and across steps (Q/K double-buffered by step, V and outputs by call)"}


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="tra", choices=["tra", "reference"])
    ap.add_argument("--workload", default="wan720")
    ap.add_argument("--calls", type=int, default=0)
    ap.add_argument("--heads", type=int, default=0, help="override the head count (smaller profiling cases)")
    ap.add_argument("--shard", default="replica", choices=["replica", "heads"],
                    help="replica: every rank runs the whole workload (weak scaling); "
                         "heads: the workload's heads are split over the ranks (strong scaling)")
    ap.add_argument("--retained", type=float, default=0.0,
                    help="target retained fraction for calibrating b (0 = the workload's own)")
    ap.add_argument("--b", type=float, default=None, help="budget offset b (default: the workload's)")
    ap.add_argument("--metric", default="square", choices=["square", "disk"],
                    help="spatial test: the Chebyshev square (default) or the Euclidean disk (TRA_FLAG_DISK)")
    ap.add_argument("--qsort", default="auto", choices=["auto", "on", "off"],
                    help="radius-sorted query groups (TRA_FLAG_QSORT): auto = when the frame has an even "
                         "number of tile columns")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-chunks", type=int, default=1,
                    help="head chunks of the end-to-end leg (each its own plan and launches)")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    raw = list(sys.argv[1:] if argv is None else argv)
    args = ap.parse_args(raw)
    if args.warmup < 3:
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        return relaunch(raw, args.gpus)
    rank, world = dist_setup(args.gpus if "WORLD_SIZE" in os.environ else 0)
    try:
        if args.impl == "reference":
            return run_reference(args, rank, world)
        line = run_tra(args, rank, world)
        if rank == 0:
            print(json.dumps(line), flush=True)
        return 0
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
