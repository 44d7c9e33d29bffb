"""Pins for the oracle's calibration quantity k_i(mass): the fewest of a
query's highest-probability keys whose dense softmax probabilities sum to at
least `mass` ("Token Radius Attention for Efficient Video Generation",
gist.science summary, section 2, Intuition I: the key density a query needs
follows its entropy).

Closed forms (uniform attention; one dominant key among equal others), the
independent numpy sort in tests/bruteforce.py, and monotonicity in the mass."""
import math

import numpy as np
import pytest

import oracle
import bruteforce as bf


def test_uniform_attention_needs_ceil_mass_times_n():
    T, H, W, d = 4, 8, 8, 16
    N = T * H * W
    q = np.zeros((1, N, d))
    k = np.random.default_rng(0).standard_normal((1, N, d))
    for mass in (0.1, 0.55, 0.9, 0.95, 0.999):
        assert mass * N != int(mass * N)
        got = oracle.topk_count(q, k, 1, (T, H, W), d, mass, queries=[0, 17, N - 1])
        assert np.all(got == math.ceil(mass * N))


def test_one_dominant_key_closed_form():
    """Scores: S for key 0, 0 for every other key, so p0 = e^S / (e^S + N - 1)
    and every other key has p1 = 1 / (e^S + N - 1)."""
    T, H, W, d = 2, 4, 8, 16
    N = T * H * W
    S = 3.0
    q = np.zeros((1, N, d))
    q[0, :, 0] = S * math.sqrt(d)
    k = np.zeros((1, N, d))
    k[0, 0, 0] = 1.0
    k[0, 1:, 1:] = np.random.default_rng(1).standard_normal((N - 1, d - 1))   # orthogonal to q
    den = math.exp(S) + N - 1
    p0, p1 = math.exp(S) / den, 1.0 / den
    for mass in (0.1, p0 - 1e-6, p0 + 1e-6, 0.5, 0.8, 0.97):
        expect = 1 if p0 >= mass else 1 + math.ceil((mass - p0) / p1 - 1e-9)
        got = oracle.topk_count(q, k, 1, (T, H, W), d, mass, queries=[5])
        assert got[0] == expect, (mass, got[0], expect)


@pytest.mark.parametrize("grid", [(4, 8, 8), (3, 7, 9), (2, 3, 5)])
def test_topk_matches_numpy_sort(grid):
    T, H, W = grid
    N, d, G = T * H * W, 16, 2
    rng = np.random.default_rng(sum(grid))
    q = rng.standard_normal((G, N, d)) * rng.lognormal(0, 0.7, (G, N, 1))
    k = rng.standard_normal((G, N, d))
    for mass in (0.5, 0.9, 0.99):
        got = oracle.topk_count(q, k, G, grid, d, mass).reshape(G, N)
        for g in range(G):
            np.testing.assert_array_equal(got[g], bf.topk_count(q[g], k[g], mass))


def test_topk_monotone_in_mass_and_bounded():
    T, H, W, d = 3, 7, 9, 16
    N = T * H * W
    rng = np.random.default_rng(3)
    q = rng.standard_normal((1, N, d)) * 2.0
    k = rng.standard_normal((1, N, d))
    prev = np.zeros(N, np.int64)
    for mass in (0.2, 0.4, 0.6, 0.8, 0.95, 0.999):
        cur = oracle.topk_count(q, k, 1, (T, H, W), d, mass)
        assert np.all(cur >= prev) and np.all((1 <= cur) & (cur <= N))
        prev = cur
