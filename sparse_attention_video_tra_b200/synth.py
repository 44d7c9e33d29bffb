"""Seeded synthetic attention inputs with the shapes of video-DiT 3D attention.

This module only draws random tensors; it holds none of the attention method's
arithmetic, so both the CUDA path and the CPU oracle can be fed from it.

Recipe (the pages evaluate on Wan2.1 / Wan2.2 / HunyuanVideo activations and
VBench, none of which are available here; these tensors stand in for them):

* Q, K, V ~ N(0, 1) i.i.d., layout [heads][N][d], natural frame-major token
  order n = (t*H + h)*W + w.
* K += F(t, h, w): a smooth 3D sinusoidal field per head and channel,
  F_c = 3^-1/2 * sum_{m=1..3} sin(2*pi*(alpha*t/T + beta*h/H + kappa*w/W) + phi)
  with alpha, beta, kappa drawn from {1, 2, 3} and phi ~ U[0, 2*pi).  Keys that
  are close in space-time are therefore similar, as in real video latents.
* every Q row is scaled by a temperature exp(0.5*z), z ~ N(0, 1) (lognormal
  with sigma 0.5), so per-query attention entropies spread out.

The base seed of workload ``i`` is ``SEED_BASE + i``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

SEED_BASE = 20260804


@dataclass(frozen=True)
class Workload:
    """One attention workload: grid T x H x W, heads, head dim and parameters."""
    name: str
    T: int
    H: int
    W: int
    heads: int
    d: int
    gamma: float
    Rt: int
    Bmin: int
    a: float = 1.0
    b: float | None = None          # None: calibrated for target_retained
    target_retained: float | None = None
    key_stride: int = 1             # 1 = dense warm-up entropy
    index: int = 0

    @property
    def N(self) -> int:
        return self.T * self.H * self.W

    @property
    def grid(self):
        return (self.T, self.H, self.W)


# The five attention shapes (tiny oracle case, Wan2.1-1.3B 480p, Wan2.1-14B
# 720p, HunyuanVideo 720p, 4x-length extension).  gamma/Rt/Bmin not fixed by
# the pages inherit the Wan values; see the design notes.
WORKLOADS = {
    "tiny": Workload("tiny 4x8x8, 2 heads, d=64", 4, 8, 8, 2, 64, 0.7, 2, 8, a=1.0, b=0.0, index=0),
    "wan480": Workload("Wan-1.3B-480p 21x30x52, 12 heads, d=128", 21, 30, 52, 12, 128, 0.8, 6, 8,
                       target_retained=0.15, index=1),
    # b fixed at the value whose radii keep 15.0 % of all token pairs on this
    # workload's seeded inputs (found once by bisection on the GPU entropies;
    # fixed so every run and both benchmark arms use the same plan)
    "wan720": Workload("Wan-14B-720p 21x45x80, 40 heads, d=128", 21, 45, 80, 40, 128, 0.8, 6, 8,
                       b=-1.1450672149658203, target_retained=0.15, index=2),
    "hunyuan720": Workload("HunyuanVideo-720p 33x45x80, 24 heads, d=128, every 8th key tile", 33, 45, 80,
                           24, 128, 0.8, 6, 8, target_retained=0.15, key_stride=8, index=3),
    "len4x": Workload("4x-length 132x45x80, 24 heads, d=128, every 8th key tile", 132, 45, 80, 24, 128,
                      0.7, 16, 8, target_retained=0.15, key_stride=8, index=4),
}


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def make_qkv(T, H, W, heads, d, seed, device="cpu", dtype=torch.float32):
    """Q, K, V [heads][N][d] (natural order) by the recipe above."""
    N = T * H * W
    g = _gen(device, seed)
    q = torch.randn(heads, N, d, generator=g, device=device, dtype=torch.float32)
    k = torch.randn(heads, N, d, generator=g, device=device, dtype=torch.float32)
    v = torch.randn(heads, N, d, generator=g, device=device, dtype=torch.float32)
    z = torch.randn(heads, N, 1, generator=g, device=device, dtype=torch.float32)
    q.mul_(torch.exp(0.5 * z))
    freq = torch.randint(1, 4, (3, heads, 3, d), generator=g, device=device).to(torch.float32)
    phi = torch.rand(heads, 3, d, generator=g, device=device, dtype=torch.float32) * (2 * math.pi)
    t = torch.arange(T, device=device, dtype=torch.float32) / T
    h = torch.arange(H, device=device, dtype=torch.float32) / H
    w = torch.arange(W, device=device, dtype=torch.float32) / W
    tt = t.view(T, 1, 1).expand(T, H, W).reshape(N)
    hh = h.view(1, H, 1).expand(T, H, W).reshape(N)
    ww = w.view(1, 1, W).expand(T, H, W).reshape(N)
    for gi in range(heads):          # one head at a time bounds the temporaries
        acc = torch.zeros(N, d, device=device, dtype=torch.float32)
        for m in range(3):
            arg = (tt[:, None] * freq[0, gi, m] + hh[:, None] * freq[1, gi, m]
                   + ww[:, None] * freq[2, gi, m]) * (2 * math.pi) + phi[gi, m]
            acc += torch.sin(arg)
        k[gi] += acc / math.sqrt(3.0)
    return q.to(dtype), k.to(dtype), v.to(dtype)


def make_v(T, H, W, heads, d, seed, device="cpu", dtype=torch.bfloat16):
    """A fresh V for a later call that reuses the mask (new seed per call)."""
    g = _gen(device, seed)
    return torch.randn(heads, T * H * W, d, generator=g, device=device, dtype=torch.float32).to(dtype)


def workload_qkv(wl: Workload, device="cpu", dtype=torch.bfloat16):
    return make_qkv(wl.T, wl.H, wl.W, wl.heads, wl.d, SEED_BASE + wl.index, device, dtype)
