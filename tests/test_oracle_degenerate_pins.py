"""Oracle pins on degenerate grids: one-row, one-column, single-frame and
single-token grids, against the independent dense numpy brute force
(tests/bruteforce.py), with the Chebyshev square and the Euclidean disk.

"Token Radius Attention for Efficient Video Generation" (gist.science
summary), section 2: the neighbourhood count (Intuition II, "Budget-vers-
Rayon"), the radius as the smallest reaching the budget, the OR-vote block
mask ("Noyaux CUDA Fusionnes") and attention restricted to the mask.  On
these grids the frame edge clips every neighbourhood in one or both spatial
directions and the temporal reach Rt' = min(Rt, T-1) is often 0, so a
clipping or reach mistake in the oracle shows here even where the ordinary
grids hide it.  The GPU's degenerate-grid parity tests rely on these."""
import math

import numpy as np
import pytest

import oracle
import bruteforce as bf

# (T, H, W, gamma, Rt)
GRIDS = [
    (1, 1, 9, 0.8, 2),      # one frame, one row
    (2, 1, 7, 0.7, 1),      # one-row frames
    (3, 6, 1, 0.8, 2),      # one-column frames
    (1, 4, 4, 0.6, 3),      # one frame (Rt' = 0 although Rt = 3)
    (4, 1, 1, 0.5, 2),      # a single token per frame
    (1, 1, 1, 0.8, 0),      # a single token
]
METRICS = [(oracle.CHEBYSHEV, False), (oracle.DISK, True)]


def _ids(g):
    return "x".join(map(str, g[:3])) + f"-Rt{g[4]}"


@pytest.mark.parametrize("metric,disk", METRICS, ids=["square", "disk"])
@pytest.mark.parametrize("grid", GRIDS, ids=_ids)
def test_count_and_radius_equal_bruteforce(grid, metric, disk):
    T, H, W, gamma, Rt = grid
    N = T * H * W
    rc = oracle.r_cap(T, H, W, gamma, Rt, metric=metric)
    assert rc == bf.r_cap(T, H, W, gamma, Rt, disk=disk)
    rng = np.random.default_rng(3 + N)
    t, h, w = bf.coords(T, H, W)
    for _ in range(4):
        r = rng.integers(0, rc + 2, size=N)
        M = bf.token_mask(T, H, W, gamma, Rt, r, disk=disk)
        for i in range(N):
            assert oracle.count(T, H, W, gamma, Rt, t[i], h[i], w[i], r[i], metric=metric) == M[i].sum()
    Hent = rng.uniform(0.0, math.log(max(N, 2)) + 0.5, size=N).astype(np.float32)
    for a, b, Bmin in ((1.0, 0.0, 1), (1.3, -0.4, 2), (0.7, 0.9, 1)):
        Bmin = min(Bmin, N)
        r_o, c_o, bh_o = oracle.radius(Hent, 1, (T, H, W), a, b, gamma, Rt, Bmin, metric=metric)
        r_b, c_b = bf.radius(Hent, T, H, W, a, b, gamma, Rt, Bmin, disk=disk)
        np.testing.assert_array_equal(bh_o, bf.bhat(Hent, a, b, N, Bmin))
        np.testing.assert_array_equal(r_o, r_b)
        np.testing.assert_array_equal(c_o, c_b)


@pytest.mark.parametrize("metric,disk", METRICS, ids=["square", "disk"])
@pytest.mark.parametrize("grid", GRIDS, ids=_ids)
def test_block_mask_and_attention_equal_bruteforce(grid, metric, disk):
    T, H, W, gamma, Rt = grid
    N = T * H * W
    G, d = 2, 8
    rng = np.random.default_rng(11 + N)
    rc = oracle.r_cap(T, H, W, gamma, Rt, metric=metric)
    r = rng.integers(0, rc + 1, size=G * N).astype(np.int32)
    q = rng.standard_normal((G, N, d))
    k = rng.standard_normal((G, N, d))
    v = rng.standard_normal((G, N, d))
    o = oracle.attention(q, k, v, r, G, (T, H, W), d, gamma, Rt, metric=metric).reshape(G, N, d)
    for (qt, kt) in (((1, 4), (1, 4)), ((2, 2), (2, 1)), ((4, 1), (2, 1))):
        bm = oracle.block_mask(r, G, (T, H, W), gamma, Rt, qt, kt, metric=metric)
        nQ = bm.shape[0] // G
        for g in range(G):
            M = bf.token_mask(T, H, W, gamma, Rt, r[g * N:(g + 1) * N], disk=disk)
            np.testing.assert_array_equal(bm[g * nQ:(g + 1) * nQ], bf.block_mask(M, T, H, W, qt, kt))
    for g in range(G):
        M = bf.token_mask(T, H, W, gamma, Rt, r[g * N:(g + 1) * N], disk=disk)
        np.testing.assert_allclose(o[g], bf.attention_masked(q[g], k[g], v[g], M), rtol=0, atol=1e-12)


@pytest.mark.parametrize("grid", GRIDS, ids=_ids)
def test_entropy_equals_bruteforce(grid):
    T, H, W = grid[:3]
    N = T * H * W
    G, d = 2, 16
    rng = np.random.default_rng(5 + N)
    q = rng.standard_normal((G, N, d)) * 1.5
    k = rng.standard_normal((G, N, d))
    h = oracle.entropy(q, k, G, (T, H, W), d).reshape(G, N)
    for g in range(G):
        np.testing.assert_allclose(h[g], bf.entropy_dense(q[g], k[g]), rtol=0, atol=1e-12)
    if N == 1:
        assert np.all(h == 0.0)                 # one key: p = 1, no uncertainty
