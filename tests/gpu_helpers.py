"""Helpers for the GPU parity tests: the tile-major index map (computed here,
independently of the library's permute kernel), layout conversion on the
host, mask-list decoding, and the tolerance checks.

Tolerances: radii, counts, lists and full bits bit-exact; entropy
|dH| <= 1e-3 * max(|H|, 1 nat); attention max-abs <= 1e-2 and mean-abs <= 1e-3
against the fp64 oracle on the same bf16 inputs.
"""
from __future__ import annotations

import numpy as np
import torch

ENT_REL = 1e-3
ATT_MAX = 1e-2
ATT_MEAN = 1e-3


def tile_major_index(info) -> np.ndarray:
    """nat[p] = natural token index of tile-major row p, -1 on pad rows."""
    p = np.arange(info.N_pad)
    tile, inn = p // 128, p % 128
    tpf = info.n_tiles_h * info.n_tiles_w
    t, rem = tile // tpf, tile % tpf
    tr, tc = rem // info.n_tiles_w, rem % info.n_tiles_w
    h = tr * info.tile_h + inn // info.tile_w
    w = tc * info.tile_w + inn % info.tile_w
    valid = (h < info.H) & (w < info.W)
    return np.where(valid, (t * info.H + h) * info.W + w, -1)


def to_tile_major(x_nat: torch.Tensor, info) -> torch.Tensor:
    """[G, N, ...] natural -> [G, N_pad, ...] tile-major, zeros on pad rows."""
    nat = torch.from_numpy(tile_major_index(info)).to(x_nat.device)
    valid = nat >= 0
    out = torch.zeros((x_nat.shape[0], info.N_pad) + tuple(x_nat.shape[2:]), dtype=x_nat.dtype, device=x_nat.device)
    out[:, valid] = x_nat[:, nat[valid]]
    return out


def to_natural(x_tm: torch.Tensor, info) -> torch.Tensor:
    nat = torch.from_numpy(tile_major_index(info)).to(x_tm.device)
    valid = nat >= 0
    out = torch.empty((x_tm.shape[0], info.N) + tuple(x_tm.shape[2:]), dtype=x_tm.dtype, device=x_tm.device)
    out[:, nat[valid]] = x_tm[:, valid]
    return out


def bf16_bits(x: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (the oracle's bf16 input type)."""
    return x.detach().to(torch.bfloat16).cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def dense_block_mask(plan, mask: torch.Tensor) -> np.ndarray:
    """Decode the library's lists into [G*n_tiles, n_tiles] with 0/1/3."""
    i = plan.info
    _, cnt, _, lst = plan.mask_views(mask)
    cnt = cnt.cpu().numpy()
    lst = lst.cpu().numpy().view(np.uint16)
    out = np.zeros((i.heads * i.n_tiles, i.n_tiles), np.uint8)
    for g in range(i.heads):
        for a in range(i.n_tiles):
            n = int(cnt[g, a])
            e = lst[g, a, :n].astype(np.int64)
            ids = e & 0x7FFF
            assert np.all(np.diff(ids) > 0), "list not strictly ascending"
            out[g * i.n_tiles + a, ids] = np.where(e & 0x8000, 3, 1)
    return out


def check_entropy(h_gpu: np.ndarray, h_ref: np.ndarray):
    h_gpu = np.asarray(h_gpu, np.float64)
    err = np.abs(h_gpu - h_ref)
    bound = ENT_REL * np.maximum(np.abs(h_ref), 1.0)
    assert np.all(np.isfinite(h_gpu))
    bad = err > bound
    assert not bad.any(), f"entropy: {bad.sum()} of {bad.size} over 1e-3 rel (max err {err.max():.3e})"


def check_attention(o_gpu: np.ndarray, o_ref: np.ndarray):
    o_gpu = np.asarray(o_gpu, np.float64)
    assert np.all(np.isfinite(o_gpu))
    err = np.abs(o_gpu - o_ref)
    assert err.max() <= ATT_MAX, f"attention max-abs {err.max():.3e} > {ATT_MAX}"
    assert err.mean() <= ATT_MEAN, f"attention mean-abs {err.mean():.3e} > {ATT_MEAN}"
