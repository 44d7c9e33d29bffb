"""Runs one attention workload through the C ABI: inputs resident in HBM in
tile-major order, the budget offset b calibrated to a target retained
fraction, and the hot path (entropy -> radius/mask -> attention calls).

Everything that computes runs in libtra_b200.so; this module allocates
buffers (torch), orders the calls and reads the retained-pair totals.
"""
from __future__ import annotations

import math

import torch

from . import Plan, synth


def shard_heads(heads: int, world: int, rank: int) -> tuple[int, int]:
    """Heads of one rank when a workload's heads are split over `world` GPUs:
    (first head, count).  Contiguous, disjoint, covering all heads, sizes
    differing by at most one.  Heads are independent attention problems, so
    no collective is needed on the path."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank outside the world")
    base, extra = divmod(int(heads), int(world))
    count = base + (1 if rank < extra else 0)
    first = rank * base + min(rank, extra)
    return first, count


class WorkloadRun:
    """One workload on one GPU.

    step(): entropy over the warm-up keys (dense, or every key_stride-th key
    tile), one radius/mask build, then `calls` attention calls that reuse the
    mask, each with its own V (drawn untimed at setup)."""

    def __init__(self, wl: synth.Workload, calls: int = 1, seed_offset: int = 0, device="cuda",
                 b: float | None = None, flags: int = 0):
        self.wl = wl
        self.calls = calls
        self.flags = flags
        self.device = device
        T, H, W, G, d = wl.T, wl.H, wl.W, wl.heads, wl.d
        probe = Plan(T, H, W, G, d, wl.a, 0.0, wl.gamma, wl.Rt, wl.Bmin, flags)    # sizes every buffer
        self.info = probe.info
        i = self.info
        seed = synth.SEED_BASE + wl.index + 1000 * seed_offset
        q, k, v = synth.make_qkv(T, H, W, G, d, seed, device=device, dtype=torch.bfloat16)
        self.q = probe.new_tile_major(device)
        self.k = probe.new_tile_major(device)
        probe.permute(q, self.q)
        probe.permute(k, self.k)
        self.v = []
        for c in range(calls):
            vc = v if c == 0 else synth.make_v(T, H, W, G, d, seed + 7919 * c, device=device)
            vt = probe.new_tile_major(device)
            probe.permute(vc, vt)
            self.v.append(vt)
            del vc
        del q, k, v
        self.out = probe.new_out(device)
        self.H = torch.empty(G, i.N_pad, dtype=torch.float32, device=device)
        self.mask = probe.new_mask(device)
        torch.cuda.synchronize()
        probe.entropy(self.q, self.k, self.H, wl.key_stride)
        if b is None:
            b = wl.b if wl.b is not None else self.calibrate_b(wl.target_retained)
        probe.close()
        self.b = b
        self.plan = Plan(T, H, W, G, d, wl.a, b, wl.gamma, wl.Rt, wl.Bmin, flags)
        self.plan.radius_and_mask(self.H, self.mask)
        torch.cuda.synchronize()
        self.retained_pairs = self.pairs()

    # ------------------------------------------------------------ calibration
    def retained_fraction(self, b: float) -> float:
        wl = self.wl
        p = Plan(wl.T, wl.H, wl.W, wl.heads, wl.d, wl.a, b, wl.gamma, wl.Rt, wl.Bmin, self.flags)
        p.radius_and_mask(self.H, self.mask)
        frac = float(p.mask_views(self.mask)[2].sum().item()) / (wl.heads * float(wl.N) ** 2)
        p.close()
        return frac

    def calibrate_b(self, target: float, iters: int = 40) -> float:
        """Bisection on b so the retained fraction (sum of c_i / (heads*N^2))
        hits `target`; the fraction is non-decreasing in b."""
        lo, hi = -30.0, 30.0
        for _ in range(iters):
            mid = 0.5 * (lo + hi)
            if self.retained_fraction(mid) < target:
                lo = mid
            else:
                hi = mid
            if hi - lo < 1e-4:
                break
        return 0.5 * (lo + hi)

    # ------------------------------------------------------------ readouts
    def pairs(self) -> int:
        return int(self.plan.mask_views(self.mask)[2].sum().item())

    def computed_pairs(self) -> int:
        """Token pairs the attention kernel touches: 128 x 128 per listed tile."""
        return int(self.plan.mask_views(self.mask)[1].sum().item()) * 128 * 128

    def retained_fraction_now(self) -> float:
        return self.retained_pairs / (self.wl.heads * float(self.wl.N) ** 2)

    def attention_flops(self) -> float:
        """Algorithmic FLOPs of one attention call: 4*d per retained pair
        (2*d for q.k, 2*d for p*v)."""
        return 4.0 * self.wl.d * self.retained_pairs

    def entropy_pairs(self) -> int:
        i, wl = self.info, self.wl
        n_key_tiles = -(-i.n_tiles // wl.key_stride)
        return wl.heads * i.N_pad * n_key_tiles * 128

    # ------------------------------------------------------------ the path
    def run_entropy(self, stream=None):
        self.plan.entropy(self.q, self.k, self.H, self.wl.key_stride, stream=stream)

    def run_mask(self, stream=None):
        self.plan.radius_and_mask(self.H, self.mask, stream=stream)

    def run_attention(self, c: int, stream=None):
        self.plan.attention(self.q, self.k, self.v[c], self.mask, self.out, stream=stream)

    def step(self, events=None, stream=None):
        """The whole hot path once.  events: optional list of CUDA events to
        record between phases: [start, after entropy, after mask, after call 0, ...]."""
        def rec(i):
            if events is not None:
                events[i].record(stream)
        rec(0)
        self.run_entropy(stream)
        rec(1)
        self.run_mask(stream)
        rec(2)
        for c in range(self.calls):
            self.run_attention(c, stream)
            rec(3 + c)

    def launches_per_step(self) -> int:
        return 2 + self.calls
