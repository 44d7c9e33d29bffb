"""Pins for the oracle's Euclidean-disk variant of the spatial test.

"Token Radius Attention for Efficient Video Generation" (gist.science
summary), section 2, Intuition II: the kept keys of a query form circular
neighbourhoods (a 2-D disk mask) whose radius decays with the frame
distance.  Here the disk is dh^2 + dw^2 <= s^2 with the same half-width
s = floor(r * gamma^|dt| + 1e-9) as the Chebyshev reading.

Pins: the Gauss circle counts (tests/golden/gauss_circle_counts.txt),
r_cap closed forms, the dense brute force (an independent numpy mask) for
counts, radii, block masks and attention, containment between the disk and
its inscribed and circumscribed squares, and monotonicity."""
import math
import os

import numpy as np
import pytest

import oracle
import bruteforce as bf

D = oracle.DISK
GOLD = os.path.join(os.path.dirname(__file__), "golden", "gauss_circle_counts.txt")


def _gauss_rows():
    rows = []
    for line in open(GOLD):
        if line.strip() and not line.startswith("#"):
            n, c = map(int, line.split())
            rows.append((n, c))
    return rows


@pytest.mark.parametrize("n,expected", _gauss_rows())
def test_interior_count_is_gauss_circle_number(n, expected):
    # one frame (Rt' = 0): s = r exactly; the query sits at the centre of a
    # 31 x 31 frame so no row is clipped for n <= 12
    assert oracle.count(1, 31, 31, 0.8, 4, 0, 15, 15, n, D) == expected


def test_r_cap_closed_forms():
    # one frame, 8 x 8: need s^2 >= 7^2 + 7^2 = 98, so s = r = 10
    assert oracle.r_cap(1, 8, 8, 0.7, 3, D) == 10
    assert bf.r_cap(1, 8, 8, 0.7, 3, disk=True) == 10
    # three frames, Rt' = 1, gamma 0.5: s(r, 1) = floor(r/2 + 1e-9); 5 x 9
    # needs s^2 >= 16 + 64 = 80, s = 9, r = 18
    assert oracle.r_cap(3, 5, 9, 0.5, 1, D) == 18
    # the disk cap is never below the square's
    for grid, gamma, Rt in (((4, 8, 8), 0.7, 2), ((3, 7, 9), 0.8, 1), ((2, 3, 5), 0.5, 3)):
        assert oracle.r_cap(*grid, gamma, Rt, D) >= oracle.r_cap(*grid, gamma, Rt)


@pytest.mark.parametrize("grid,gamma,Rt", [((4, 8, 8), 0.7, 2), ((3, 7, 9), 0.8, 1), ((2, 3, 5), 0.5, 3),
                                           ((2, 11, 6), 0.9, 1)])
def test_count_equals_bruteforce_mask_rows(grid, gamma, Rt):
    T, H, W = grid
    N = T * H * W
    t, h, w = bf.coords(T, H, W)
    for r in range(0, oracle.r_cap(T, H, W, gamma, Rt, D) + 2):
        M = bf.token_mask(T, H, W, gamma, Rt, np.full(N, r), disk=True)
        c = [oracle.count(T, H, W, gamma, Rt, int(t[i]), int(h[i]), int(w[i]), r, D) for i in range(N)]
        np.testing.assert_array_equal(np.array(c), M.sum(axis=1))


def test_disk_between_inscribed_and_circumscribed_squares():
    """Chebyshev half-width floor(s / sqrt 2) <= disk <= Chebyshev half-width s."""
    T, H, W, gamma, Rt = 3, 13, 17, 0.8, 1
    N = T * H * W
    rng = np.random.default_rng(0)
    r = rng.integers(0, 12, N)
    Md = bf.token_mask(T, H, W, gamma, Rt, r, disk=True)
    Mo = bf.token_mask(T, H, W, gamma, Rt, r)
    assert not (Md & ~Mo).any()
    # inscribed square: replace every radius by the one whose half-width is
    # at most s / sqrt 2 in every frame -- checked pairwise on the token test
    for i in rng.choice(N, 40, replace=False):
        for j in range(N):
            if oracle.token_mask(T, H, W, gamma, Rt, int(i), j, int(r[i]), D):
                assert oracle.token_mask(T, H, W, gamma, Rt, int(i), j, int(r[i]))
            ti, hi, wi = i // (H * W), (i // W) % H, i % W
            tj, hj, wj = j // (H * W), (j // W) % H, j % W
            dt = abs(ti - tj)
            if dt > min(Rt, T - 1):
                continue
            s = oracle.halfwidth(int(r[i]), gamma ** dt)
            if max(abs(hi - hj), abs(wi - wj)) <= math.floor(s / math.sqrt(2.0)):
                assert oracle.token_mask(T, H, W, gamma, Rt, int(i), j, int(r[i]), D)


@pytest.mark.parametrize("grid,gamma,Rt,Bmin", [((4, 8, 8), 0.7, 2, 8), ((3, 7, 9), 0.8, 1, 4),
                                                ((2, 3, 5), 0.5, 3, 2)])
def test_radius_matches_bruteforce(grid, gamma, Rt, Bmin):
    T, H, W = grid
    N = T * H * W
    rng = np.random.default_rng(7)
    for a, b in ((1.0, 0.0), (1.0, 1.5), (0.5, -0.5)):
        Hent = rng.uniform(0.0, math.log(N), N).astype(np.float32)
        r_o, c_o, bh_o = oracle.radius(Hent, 1, grid, a, b, gamma, Rt, Bmin, metric=D)
        r_b, c_b = bf.radius(Hent, T, H, W, a, b, gamma, Rt, Bmin, disk=True)
        np.testing.assert_array_equal(bh_o, bf.bhat(Hent, a, b, N, Bmin))
        np.testing.assert_array_equal(r_o, r_b)
        np.testing.assert_array_equal(c_o, c_b)


def test_radius_minimal_and_monotone():
    T, H, W, gamma, Rt, Bmin = 3, 9, 11, 0.8, 1, 3
    N = T * H * W
    t, h, w = bf.coords(T, H, W)
    rng = np.random.default_rng(1)
    Hent = rng.uniform(0.0, math.log(N), N).astype(np.float32)
    r, c, bh = oracle.radius(Hent, 1, (T, H, W), 1.0, 0.0, gamma, Rt, Bmin, metric=D)
    for i in range(N):
        if r[i] > 0:
            assert oracle.count(T, H, W, gamma, Rt, int(t[i]), int(h[i]), int(w[i]), int(r[i]) - 1, D) < bh[i]
        assert c[i] >= min(bh[i], N) or r[i] == oracle.r_cap(T, H, W, gamma, Rt, D)
        for rr in range(1, 6):
            assert (oracle.count(T, H, W, gamma, Rt, int(t[i]), int(h[i]), int(w[i]), rr, D) >=
                    oracle.count(T, H, W, gamma, Rt, int(t[i]), int(h[i]), int(w[i]), rr - 1, D))


@pytest.mark.parametrize("grid,qt,kt", [((4, 8, 8), (8, 16), (8, 16)), ((3, 7, 9), (2, 4), (2, 4)),
                                        ((2, 9, 13), (4, 4), (2, 8))])
def test_block_mask_matches_bruteforce(grid, qt, kt):
    T, H, W = grid
    N = T * H * W
    gamma, Rt = 0.8, 2
    rng = np.random.default_rng(3)
    r = rng.integers(0, 9, N).astype(np.int32)
    bm = oracle.block_mask(r, 1, grid, gamma, Rt, qt, kt, metric=D)
    M = bf.token_mask(T, H, W, gamma, Rt, r, disk=True)
    np.testing.assert_array_equal(bm, bf.block_mask(M, T, H, W, qt, kt))


@pytest.mark.parametrize("grid,gamma,Rt", [((4, 8, 8), 0.7, 2), ((3, 7, 9), 0.8, 1)])
def test_attention_matches_bruteforce(grid, gamma, Rt):
    T, H, W = grid
    N, d, G = T * H * W, 16, 2
    rng = np.random.default_rng(5)
    q, k, v = (rng.standard_normal((G, N, d)) for _ in range(3))
    r = rng.integers(0, 6, G * N).astype(np.int32)
    o = oracle.attention(q, k, v, r, G, grid, d, gamma, Rt, metric=D).reshape(G, N, d)
    for g in range(G):
        M = bf.token_mask(T, H, W, gamma, Rt, r[g * N:(g + 1) * N], disk=True)
        np.testing.assert_allclose(o[g], bf.attention_masked(q[g], k[g], v[g], M), rtol=0, atol=1e-12)


def test_metric_zero_is_the_default_reading():
    T, H, W, gamma, Rt = 3, 7, 9, 0.8, 1
    assert oracle.count(T, H, W, gamma, Rt, 1, 3, 4, 5) == oracle.count(T, H, W, gamma, Rt, 1, 3, 4, 5, oracle.CHEBYSHEV)
    # at s = 1 the disk drops exactly the four diagonal neighbours of the square
    assert oracle.count(1, 9, 9, 0.8, 0, 0, 4, 4, 1) - oracle.count(1, 9, 9, 0.8, 0, 0, 4, 4, 1, D) == 4
