"""Pins for the oracle's radius-sorted query groups (the library's
TRA_FLAG_QSORT plans; a scheduling design of this library, not of the pages)
and for the block mask of explicit query sets.

* Block masks of sets equal the tile block mask when the sets are the tiles
  (two independent oracle paths), and a dense numpy brute force for arbitrary
  sets (bruteforce.token_mask).
* The groups of a strip (one tile column of one frame) partition its
  128*nTh rows, radii never decrease from one group to the next or inside a
  group, equal radii keep row order, and pad rows come first.
* Token voting is an OR, so the union of a strip's groups' active tiles
  equals the union of the strip's tiles' active tiles."""
import numpy as np
import pytest

import oracle
import bruteforce as bf


def _tile_members(G, grid, tile):
    T, H, W = grid
    th, tw = tile
    nTh, nTw = -(-H // th), -(-W // tw)
    nQ = T * nTh * nTw
    N = T * H * W
    mem = np.full((G * nQ, 128), -1, np.int64)
    for g in range(G):
        for a in range(nQ):
            t, rem = a // (nTh * nTw), a % (nTh * nTw)
            for i in range(128):
                h = (rem // nTw) * th + i // tw
                w = (rem % nTw) * tw + i % tw
                if h < H and w < W:
                    mem[g * nQ + a, i] = g * N + (t * H + h) * W + w
    return mem


@pytest.mark.parametrize("grid,tile,metric", [((4, 8, 8), (16, 8), oracle.CHEBYSHEV), ((3, 7, 9), (8, 16), oracle.CHEBYSHEV),
                                              ((2, 9, 13), (4, 32), oracle.DISK)])
def test_sets_equal_tiles_when_sets_are_tiles(grid, tile, metric):
    T, H, W = grid
    G, N = 2, T * H * W
    for lo, hi in ((0, 7), (40, 41)):      # mixed small radii; radii that make every reachable tile full
        r = np.random.default_rng(1).integers(lo, hi, G * N).astype(np.int32)
        mem = _tile_members(G, grid, tile)
        a = oracle.block_mask_sets(r, G, grid, 0.8, 2, tile, mem, metric=metric)
        b = oracle.block_mask(r, G, grid, 0.8, 2, tile, tile, metric=metric)
        np.testing.assert_array_equal(a, b)
        if lo == 40:
            assert (b == 3).any()


@pytest.mark.parametrize("disk", [False, True])
def test_sets_equal_bruteforce(disk):
    T, H, W, gamma, Rt = 3, 7, 9, 0.8, 1
    N = T * H * W
    rng = np.random.default_rng(2)
    kt = (2, 4)
    kid, nK = bf.tile_ids(T, H, W, *kt)
    n_full = 0
    for lo, hi in ((0, 6), (20, 30)):      # small radii; radii that make full tiles
        r = rng.integers(lo, hi, N).astype(np.int32)
        M = bf.token_mask(T, H, W, gamma, Rt, r, disk=disk)        # [N, N] keep
        sets = np.full((6, 10), -1, np.int64)
        for s in range(6):
            k = rng.integers(1, 11)
            sets[s, :k] = rng.choice(N, size=k, replace=False)
        got = oracle.block_mask_sets(r, 1, (T, H, W), gamma, Rt, kt, sets,
                                     metric=oracle.DISK if disk else oracle.CHEBYSHEV)
        for s in range(6):
            q = sets[s][sets[s] >= 0]
            for kb in range(nK):
                keys = np.nonzero(kid == kb)[0]
                blk = M[np.ix_(q, keys)]
                want = (3 if blk.all() else 1) if blk.any() else 0
                n_full += want == 3
                assert got[s, kb] == want
    assert n_full > 0


def _strip_tiles(grid, tile):
    T, H, W = grid
    th, tw = tile
    nTh, nTw = -(-H // th), -(-W // tw)
    return [[t * nTh * nTw + u * nTw + c for u in range(nTh)] for t in range(T) for c in range(nTw)]


@pytest.mark.parametrize("grid,tile", [((3, 20, 16), (16, 8)), ((2, 45, 80), (16, 8)), ((2, 30, 20), (8, 16)),
                                       ((3, 8, 12), (32, 4))])
def test_groups_partition_strips_sorted_by_radius(grid, tile):
    T, H, W = grid
    G = 2
    N = T * H * W
    r = np.random.default_rng(3).integers(0, 9, G * N).astype(np.int32)
    perm, mem = oracle.query_groups(r, G, grid, tile)
    nQ = perm.shape[1]
    tm = _tile_members(G, grid, tile)
    for g in range(G):
        for tiles in _strip_tiles(grid, tile):
            U = len(tiles)
            allp = np.concatenate([perm[g, a] for a in tiles]).astype(np.int64)
            assert sorted(allp.tolist()) == list(range(128 * U))
            strip_rows = np.concatenate([tm[g * nQ + a] for a in tiles])
            rad = np.where(strip_rows >= 0, r[np.maximum(strip_rows, 0)], -1)
            ordered = rad[allp]
            assert np.all(np.diff(ordered) >= 0)                     # sorted by radius (pads, -1, first)
            for v in np.unique(ordered):
                rows = allp[ordered == v]
                assert np.all(np.diff(rows) > 0)                     # ties keep row order
            for u, a in enumerate(tiles):
                np.testing.assert_array_equal(mem[g * nQ + a], strip_rows[perm[g, a].astype(np.int64)])


@pytest.mark.parametrize("grid,tile", [((3, 20, 16), (16, 8)), ((2, 30, 20), (8, 16))])
def test_group_union_equals_tile_union(grid, tile):
    T, H, W = grid
    G = 2
    N = T * H * W
    r = np.random.default_rng(4).integers(0, 9, G * N).astype(np.int32)
    _, mem = oracle.query_groups(r, G, grid, tile)
    grp = oracle.block_mask_sets(r, G, grid, 0.8, 2, tile, mem) > 0
    til = oracle.block_mask(r, G, grid, 0.8, 2, tile, tile) > 0
    nQ = grp.shape[0] // G
    for g in range(G):
        for tiles in _strip_tiles(grid, tile):
            rows = [g * nQ + a for a in tiles]
            np.testing.assert_array_equal(np.any(grp[rows], axis=0), np.any(til[rows], axis=0))
