"""Pins for the oracle's calibration quantity k_i(mass): the fewest of a
query's highest-probability keys whose dense softmax probabilities sum to at
least `mass` ("Token Radius Attention for Efficient Video Generation",
gist.science summary, section 2, Intuition I: the key density a query needs
follows its entropy).

Closed forms (uniform attention; one dominant key among equal others), the
independent numpy sort in tests/bruteforce.py, and monotonicity in the mass.

The fit ln k = a*H + b that turns those pairs into the plan's budget
constants is pinned by a hand-worked three-point case, the line through two
points, exact recovery of a known (a, b), and numpy.polyfit on noisy data."""
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


# ---------------------------------------------------------------- the fit ln k = a*H + b
def test_fit_hand_worked_three_points():
    """x = H = (0, 1, 2), k = (1, 2, 8): y = ln k = (0, 1, 3)*ln 2.  By hand:
    mean x = 1, mean y = (4/3) ln 2, S_xy = 3 ln 2, S_xx = 2, so
    a = (3/2) ln 2 and b = (4/3 - 3/2) ln 2 = -(1/6) ln 2; S_yy = (42/9) ln^2 2,
    r2 = 9 ln^2 2 / (2 * 42/9 ln^2 2) = 81/84."""
    a, b, r2, m = oracle.fit_log_linear([0.0, 1.0, 2.0], [1, 2, 8])
    L2 = math.log(2.0)
    assert m == 3
    assert a == pytest.approx(1.5 * L2, rel=1e-14)
    assert b == pytest.approx(-L2 / 6.0, rel=1e-13)
    assert r2 == pytest.approx(81.0 / 84.0, rel=1e-14)


def test_fit_two_points_is_the_line_through_them():
    H1, H2, k1, k2 = 1.25, 4.0, 3, 170
    a, b, r2, m = oracle.fit_log_linear([H1, H2], [k1, k2])
    slope = (math.log(k2) - math.log(k1)) / (H2 - H1)
    assert a == pytest.approx(slope, rel=1e-14)
    assert b == pytest.approx(math.log(k1) - slope * H1, rel=1e-13, abs=1e-14)
    assert r2 == pytest.approx(1.0, rel=1e-14)


def test_fit_recovers_exact_log_linear_data():
    """H_i placed exactly on ln k = 1.3*H - 0.5 for integer k_i (the tau*exp(H)
    law with slope 1.3): the fit returns (1.3, -0.5)."""
    rng = np.random.default_rng(11)
    k = rng.integers(1, 5000, 400)
    H = (np.log(k) + 0.5) / 1.3
    a, b, r2, m = oracle.fit_log_linear(H, k)
    assert m == 400
    assert a == pytest.approx(1.3, abs=1e-12)
    assert b == pytest.approx(-0.5, abs=1e-11)
    assert r2 == pytest.approx(1.0, abs=1e-12)


def test_fit_matches_numpy_polyfit_on_noisy_data():
    """Against an independent least-squares routine (numpy.polyfit, degree 1)."""
    rng = np.random.default_rng(12)
    H = rng.uniform(2.0, 10.0, 3000)
    k = np.maximum(1, np.round(np.exp(0.9 * H + 0.7 + rng.normal(0, 0.6, H.size)))).astype(np.int64)
    a, b, r2, m = oracle.fit_log_linear(H, k)
    pa, pb = np.polyfit(H, np.log(k), 1)
    assert a == pytest.approx(pa, rel=1e-10)
    assert b == pytest.approx(pb, rel=1e-10, abs=1e-10)
    assert 0.5 < r2 < 1.0


def test_fit_ignores_unusable_rows_and_rejects_degenerate_input():
    H = [0.0, 1.0, 2.0, float("nan"), 5.0, float("inf")]
    k = [1, 2, 8, 40, 0, 7]          # the NaN-H, k=0 and inf-H rows are not used
    a, b, r2, m = oracle.fit_log_linear(H, k)
    assert m == 3 and a == pytest.approx(1.5 * math.log(2.0), rel=1e-14)
    with pytest.raises(ValueError):
        oracle.fit_log_linear([1.0, 2.0], [5, -1])          # one usable row
    with pytest.raises(ValueError):
        oracle.fit_log_linear([3.0, 3.0, 3.0], [1, 5, 9])   # no spread in H
