"""CPU pins of the fp64 oracle against things other than itself: hand-derived
closed forms, invariants, special cases that reduce to a library routine, and
an independent dense numpy brute force on tiny grids.

Definitions: "Token Radius Attention for Efficient Video Generation"
(gist.science summary), section 2 (Intuition I: entropy -> budget; Intuition II:
query-centred radius with temporal decay; "Le Pipeline TRA").
"""
import math
import os

import numpy as np
import pytest
import torch

import bruteforce as bf
import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "closed_form_counts.txt")


def _rand_qkv(G, N, d, seed, temp=True):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((G, N, d))
    k = rng.standard_normal((G, N, d))
    v = rng.standard_normal((G, N, d))
    if temp:
        q *= np.exp(0.5 * rng.standard_normal((G, N, 1)))
    return q, k, v


# ----------------------------------------------------------------- half-width
def test_halfwidth_closed_forms():
    # gamma^0 = 1: s = r exactly
    for r in range(0, 2000, 7):
        assert oracle.halfwidth(r, 1.0) == r
    assert oracle.halfwidth(0, 0.37) == 0
    # 25*0.8^2 is 16.000000000000004 in fp64: floor -> 16
    assert oracle.halfwidth(25, math.pow(0.8, 2)) == 16
    # 100*0.7^2 is 48.99999999999999 in fp64: the 1e-9 lifts it to 49
    assert oracle.halfwidth(100, math.pow(0.7, 2)) == 49
    # 3*0.7 = 2.0999999999999996 -> 2 ; 3*0.49 -> 1
    assert oracle.halfwidth(3, 0.7) == 2
    assert oracle.halfwidth(3, math.pow(0.7, 2)) == 1


def test_decay_table_is_powers():
    g = oracle.decay_table(0.8, 6)
    assert g[0] == 1.0
    for k in range(1, 7):
        assert g[k] == math.pow(0.8, k)
        assert g[k] < g[k - 1]


def test_rt_eff_and_r_cap():
    assert oracle.rt_eff(2, 5) == 1
    assert oracle.rt_eff(21, 6) == 6
    # T=4,H=W=8, gamma=0.7, Rt=2: need floor(r*0.49+1e-9) >= 7 -> r = 15 (14*0.49=6.86)
    assert oracle.r_cap(4, 8, 8, 0.7, 2) == 15
    # single frame: Rt'=0, g=1, need s = r >= max(H,W)-1
    assert oracle.r_cap(1, 5, 9, 0.5, 3) == 8
    assert oracle.r_cap(1, 1, 1, 0.5, 3) == 0


# ----------------------------------------------------------------- counts
def _golden_rows():
    rows = []
    for line in open(GOLDEN):
        line = line.split("#")[0].strip()
        if line:
            f = line.split()
            rows.append(tuple(int(x) if i != 3 else float(x) for i, x in enumerate(f)))
    return rows


@pytest.mark.parametrize("row", _golden_rows())
def test_count_golden(row):
    T, H, W, gamma, Rt, t, h, w, r, expect = row
    assert oracle.count(T, H, W, gamma, Rt, t, h, w, r) == expect


def test_count_interior_formula():
    # interior query: c = sum_dt (2 s(r,|dt|) + 1)^2 over 2Rt+1 frames
    T, H, W, gamma, Rt = 15, 61, 61, 0.8, 3
    for r in range(0, 25):
        s = [oracle.halfwidth(r, math.pow(gamma, k)) for k in range(Rt + 1)]
        expect = (2 * s[0] + 1) ** 2 + 2 * sum((2 * s[k] + 1) ** 2 for k in range(1, Rt + 1))
        assert oracle.count(T, H, W, gamma, Rt, 7, 30, 30, r) == expect


@pytest.mark.parametrize("grid,gamma,Rt", [((4, 8, 8), 0.7, 2), ((3, 7, 9), 0.8, 1),
                                          ((5, 4, 6), 0.5, 4), ((2, 3, 5), 0.9, 0)])
def test_count_equals_bruteforce_mask_rows(grid, gamma, Rt):
    T, H, W = grid
    N = T * H * W
    rng = np.random.default_rng(1)
    rc = oracle.r_cap(T, H, W, gamma, Rt)
    for _ in range(6):
        r = rng.integers(0, rc + 1, size=N)
        M = bf.token_mask(T, H, W, gamma, Rt, r)
        t, h, w = bf.coords(T, H, W)
        for i in range(N):
            assert oracle.count(T, H, W, gamma, Rt, t[i], h[i], w[i], r[i]) == M[i].sum()


def test_count_monotone_in_r_and_reaches_all_at_rcap():
    T, H, W, gamma, Rt = 6, 9, 11, 0.6, 5
    rc = oracle.r_cap(T, H, W, gamma, Rt)
    t, h, w = bf.coords(T, H, W)
    for i in range(0, T * H * W, 13):
        cs = [oracle.count(T, H, W, gamma, Rt, t[i], h[i], w[i], r) for r in range(rc + 3)]
        assert all(a <= b for a, b in zip(cs, cs[1:]))
        assert cs[rc] == T * H * W  # Rt' = T-1 here: the full grid
        assert cs[rc + 2] == cs[rc]


# ----------------------------------------------------------------- budget
def test_budget_closed_forms():
    N = 1000
    assert oracle.budget(0.0, 1.0, 0.0, N, 8) == 8                       # exp(0)=1 < Bmin
    assert oracle.budget(20.0, 1.0, 0.0, N, 8) == N                      # clamp at N
    assert oracle.budget(float(np.float32(math.log(100.5))), 1.0, 0.0, N, 8) == 101
    assert oracle.budget(3.7, 0.0, math.log(50.5), N, 1) == 51            # a = 0: one shared budget
    assert oracle.budget(-5.0, 1.0, 0.0, N, 1) == 1                      # exp(-5) -> ceil -> 1
    # tau*exp(H) form: a = 1, b = ln tau
    assert oracle.budget(float(np.float32(math.log(41.0))), 1.0, math.log(0.5), N, 1) == 21  # 20.5 -> 21


def test_budget_monotone_in_entropy():
    Hs = np.linspace(0, 8, 400).astype(np.float32)
    for a in (0.5, 1.0, 1.7):
        bs = [oracle.budget(float(x), a, -1.0, 5000, 4) for x in Hs]
        assert all(x <= y for x, y in zip(bs, bs[1:]))


# ----------------------------------------------------------------- radius
@pytest.mark.parametrize("grid,gamma,Rt,Bmin", [((4, 8, 8), 0.7, 2, 8), ((3, 7, 9), 0.8, 1, 4),
                                               ((2, 3, 5), 0.5, 3, 1)])
def test_radius_matches_bruteforce(grid, gamma, Rt, Bmin):
    T, H, W = grid
    N = T * H * W
    rng = np.random.default_rng(7)
    Hent = rng.uniform(0.0, math.log(N) + 0.5, size=N).astype(np.float32)
    for a, b in ((1.0, 0.0), (1.3, -0.7), (0.8, 0.9)):
        r_o, c_o, bh_o = oracle.radius(Hent, 1, grid, a, b, gamma, Rt, Bmin)
        r_b, c_b = bf.radius(Hent, T, H, W, a, b, gamma, Rt, Bmin)
        np.testing.assert_array_equal(bh_o, bf.bhat(Hent, a, b, N, Bmin))
        np.testing.assert_array_equal(r_o, r_b)
        np.testing.assert_array_equal(c_o, c_b)


def test_radius_sampled_rows_equal_full():
    T, H, W = 5, 6, 7
    N = T * H * W
    Hent = np.random.default_rng(3).uniform(0, 5, size=2 * N).astype(np.float32)
    r, c, _ = oracle.radius(Hent, 2, (T, H, W), 1.0, 0.2, 0.8, 2, 3)
    idx = np.array([0, 5, N - 1, N, 2 * N - 1, 77])
    r2, c2, _ = oracle.radius(Hent[idx], 2, (T, H, W), 1.0, 0.2, 0.8, 2, 3, queries=idx)
    np.testing.assert_array_equal(r2, r[idx])
    np.testing.assert_array_equal(c2, c[idx])


def test_radius_monotone_in_budget_at_fixed_position():
    T, H, W = 5, 9, 9
    N = T * H * W
    Hs = np.linspace(0, math.log(N), 64).astype(np.float32)
    for pos in (0, N // 2, 17):
        idx = np.full(Hs.size, pos)
        r, c, bh = oracle.radius(Hs, 1, (T, H, W), 1.0, 0.0, 0.7, 2, 1, queries=idx)
        assert np.all(np.diff(bh) >= 0) and np.all(np.diff(r) >= 0)
        # minimality: the count reaches the budget, one step less does not
        t, h, w = bf.coords(T, H, W)
        for rr, cc, b in zip(r, c, bh):
            if cc >= b and rr > 0:
                assert oracle.count(T, H, W, 0.7, 2, t[pos], h[pos], w[pos], rr - 1) < b


def test_self_only_case():
    # Rt = 0, Bmin = 1, tiny budget -> r = 0, c = 1, O_i = v_i
    T, H, W, d, G = 3, 5, 6, 8, 2
    N = T * H * W
    q, k, v = _rand_qkv(G, N, d, 11)
    Hent = np.full(G * N, 2.0, np.float32)
    r, c, _ = oracle.radius(Hent, G, (T, H, W), 1.0, -1000.0, 0.8, 0, 1)
    assert np.all(r == 0) and np.all(c == 1)
    o = oracle.attention(q, k, v, r, G, (T, H, W), d, 0.8, 0)
    np.testing.assert_allclose(o.reshape(G, N, d), v, rtol=0, atol=1e-15)


def test_dense_case_equals_sdpa():
    # Rt = T-1 and Bhat = N -> r = r_cap, every query keeps all N keys,
    # so the masked attention is plain softmax attention (torch SDPA, fp64).
    T, H, W, d, G = 3, 4, 5, 16, 2
    N = T * H * W
    q, k, v = _rand_qkv(G, N, d, 5)
    Hent = np.full(G * N, 1.0, np.float32)
    r, c, bh = oracle.radius(Hent, G, (T, H, W), 1.0, 50.0, 0.7, T - 1, 1)
    assert np.all(bh == N) and np.all(c == N)
    # smallest radius reaching all N keys: never above r_cap; corners need r_cap
    assert np.all(r <= oracle.r_cap(T, H, W, 0.7, T - 1))
    assert r[0] == oracle.r_cap(T, H, W, 0.7, T - 1)
    o = oracle.attention(q, k, v, r, G, (T, H, W), d, 0.7, T - 1).reshape(G, N, d)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(k)[None], torch.from_numpy(v)[None])[0].numpy()
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)


# ----------------------------------------------------------------- entropy
def test_entropy_two_point_closed_form():
    # 2 keys, scores (0, ln 3): p = (1/4, 3/4), H = ln 4 - (3/4) ln 3
    d = 4
    q = np.zeros((1, 2, d)); q[0, :, 0] = 2.0          # sigma = 1/2
    k = np.zeros((1, 2, d)); k[0, 1, 0] = math.log(3.0)
    h = oracle.entropy(q, k, 1, (1, 1, 2), d)
    expect = math.log(4.0) - 0.75 * math.log(3.0)
    assert abs(h[0] - expect) < 1e-14
    # query 1 sees the same scores
    assert abs(h[1] - expect) < 1e-14


def test_entropy_uniform_and_peaked():
    G, T, H, W, d = 1, 2, 3, 4, 8
    N = T * H * W
    rng = np.random.default_rng(2)
    k = rng.standard_normal((G, N, d))
    q0 = np.zeros((G, N, d))
    h0 = oracle.entropy(q0, k, G, (T, H, W), d)
    np.testing.assert_allclose(h0, math.log(N), rtol=0, atol=1e-13)
    # one key far ahead: entropy -> 0
    kk = np.zeros((G, N, d)); kk[0, 5, 0] = 1.0
    qq = np.zeros((G, N, d)); qq[..., 0] = 400.0 * math.sqrt(d)
    h1 = oracle.entropy(qq, kk, G, (T, H, W), d)
    assert np.all(h1 < 1e-100 + 1e-12) and np.all(h1 >= -1e-15)


def test_entropy_q_zero_subsampled_keeps_log_n():
    # Q = 0: the sampled plug-in entropy is ln|S|, the correction makes it ln N
    G, T, H, W, d = 2, 4, 8, 8, 8
    N = T * H * W
    k = np.random.default_rng(4).standard_normal((G, N, d))
    q0 = np.zeros((G, N, d))
    for stride, kt in ((8, (2, 4)), (3, (4, 8)), (2, (8, 8))):
        h = oracle.entropy(q0, k, G, (T, H, W), d, key_stride=stride, ktile=kt)
        np.testing.assert_allclose(h, math.log(N), rtol=0, atol=1e-12)


@pytest.mark.parametrize("grid", [(4, 8, 8), (3, 7, 9), (2, 3, 5)])
def test_entropy_matches_bruteforce(grid):
    T, H, W = grid
    N = T * H * W
    G, d = 2, 16
    q, k, _ = _rand_qkv(G, N, d, 9)
    h = oracle.entropy(q, k, G, grid, d).reshape(G, N)
    for g in range(G):
        np.testing.assert_allclose(h[g], bf.entropy_dense(q[g], k[g]), rtol=0, atol=1e-12)


def test_entropy_subsampled_matches_bruteforce():
    T, H, W = 4, 8, 8
    N = T * H * W
    G, d = 1, 8
    q, k, _ = _rand_qkv(G, N, d, 13)
    kid, _ = bf.tile_ids(T, H, W, 2, 8)
    sel = np.nonzero(kid % 3 == 0)[0]
    h = oracle.entropy(q, k, G, (T, H, W), d, key_stride=3, ktile=(2, 8))
    ref = bf.entropy_dense(q[0], k[0][sel]) + math.log(N / sel.size)
    np.testing.assert_allclose(h, ref, rtol=0, atol=1e-12)


def test_entropy_bf16_and_f32_inputs_agree_with_f64():
    G, T, H, W, d = 1, 2, 4, 4, 8
    N = T * H * W
    rng = np.random.default_rng(5)
    x = rng.standard_normal((2, G, N, d)).astype(np.float32)
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)          # truncated bf16
    back = (bits.astype(np.uint32) << 16).view(np.float32)
    h16 = oracle.entropy(bits[0], bits[1], G, (T, H, W), d)
    h64 = oracle.entropy(back[0].astype(np.float64), back[1].astype(np.float64), G, (T, H, W), d)
    h32 = oracle.entropy(back[0], back[1], G, (T, H, W), d)
    np.testing.assert_array_equal(h16, h64)
    np.testing.assert_array_equal(h32, h64)


# ----------------------------------------------------------------- attention
@pytest.mark.parametrize("grid,gamma,Rt", [((4, 8, 8), 0.7, 2), ((3, 7, 9), 0.8, 1), ((2, 3, 5), 0.5, 3)])
def test_attention_matches_bruteforce(grid, gamma, Rt):
    T, H, W = grid
    N = T * H * W
    G, d = 2, 16
    q, k, v = _rand_qkv(G, N, d, 21)
    rng = np.random.default_rng(8)
    rc = oracle.r_cap(T, H, W, gamma, Rt)
    r = rng.integers(0, rc + 1, size=G * N).astype(np.int32)
    o = oracle.attention(q, k, v, r, G, grid, d, gamma, Rt).reshape(G, N, d)
    for g in range(G):
        M = bf.token_mask(T, H, W, gamma, Rt, r[g * N:(g + 1) * N])
        np.testing.assert_allclose(o[g], bf.attention_masked(q[g], k[g], v[g], M), rtol=0, atol=1e-12)


def test_attention_sampled_rows_equal_full():
    T, H, W = 3, 5, 5
    N = T * H * W
    G, d = 2, 8
    q, k, v = _rand_qkv(G, N, d, 2)
    r = np.random.default_rng(1).integers(0, 6, size=G * N).astype(np.int32)
    full = oracle.attention(q, k, v, r, G, (T, H, W), d, 0.8, 2)
    idx = np.array([3, N + 7, 2 * N - 1])
    part = oracle.attention(q, k, v, r, G, (T, H, W), d, 0.8, 2, queries=idx)
    np.testing.assert_array_equal(part, full[idx])


# ----------------------------------------------------------------- block mask
@pytest.mark.parametrize("grid,qt,kt", [((4, 8, 8), (8, 16), (8, 16)), ((3, 7, 9), (2, 4), (2, 4)),
                                        ((3, 7, 9), (4, 2), (2, 2)), ((2, 5, 6), (2, 2), (1, 2)),
                                        ((4, 8, 8), (4, 4), (2, 4))])
def test_block_mask_matches_bruteforce(grid, qt, kt):
    T, H, W = grid
    N = T * H * W
    gamma, Rt = 0.7, 2
    rng = np.random.default_rng(17)
    rc = oracle.r_cap(T, H, W, gamma, Rt)
    r = rng.integers(0, rc + 1, size=N).astype(np.int32)
    r[rng.random(N) < 0.3] = 0
    bm = oracle.block_mask(r, 1, grid, gamma, Rt, qt, kt)
    M = bf.token_mask(T, H, W, gamma, Rt, r)
    np.testing.assert_array_equal(bm, bf.block_mask(M, T, H, W, qt, kt))
    # every retained token pair lies in an active tile pair (skipping inactive
    # tiles never changes the output)
    qid, _ = bf.tile_ids(T, H, W, *qt)
    kid, _ = bf.tile_ids(T, H, W, *kt)
    ii, jj = np.nonzero(M)
    assert np.all(bm[qid[ii], kid[jj]] & 1)
    # the query's own tile pair is always active (each query keeps itself)
    own = bm[qid, kid]
    assert np.all(own & 1)


def test_block_mask_sampled_rows_equal_full():
    T, H, W = 3, 6, 8
    r = np.random.default_rng(0).integers(0, 9, size=2 * T * H * W).astype(np.int32)
    full = oracle.block_mask(r, 2, (T, H, W), 0.8, 1, (2, 4), (2, 4))
    idx = np.array([0, 5, full.shape[0] - 1, 13])
    part = oracle.block_mask(r, 2, (T, H, W), 0.8, 1, (2, 4), (2, 4), qtiles=idx)
    np.testing.assert_array_equal(part, full[idx])


def test_temporal_limit_never_exceeded():
    # keys beyond Rt frames are never attended, whatever the radius
    T, H, W, gamma, Rt = 7, 4, 4, 0.9, 2
    N = T * H * W
    r = np.full(N, 10_000, np.int32)
    t, h, w = bf.coords(T, H, W)
    for i in range(0, N, 5):
        for j in range(N):
            m = oracle.token_mask(T, H, W, gamma, Rt, i, j, int(r[i]))
            assert m == (abs(int(t[i]) - int(t[j])) <= Rt)
