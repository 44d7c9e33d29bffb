"""GPU parity for the Euclidean-disk spatial test (TRA_FLAG_DISK) against the
oracle's metric 1.

"Token Radius Attention for Efficient Video Generation" (gist.science
summary), section 2, Intuition II: circular neighbourhoods (a 2-D disk mask)
with a radius that decays with the frame distance.  Same half-width s as the
Chebyshev reading; the test is dh^2 + dw^2 <= s^2.

Radii, retained-pair totals and block masks (lists and full bits) are
bit-exact given the same entropies; attention is within the usual max-abs
1e-2 / mean-abs 1e-3 of the fp64 oracle; the natural-layout path matches the
tile-major one bit for bit."""
import math

import numpy as np
import pytest
import torch

import oracle
import sparse_attention_video_tra_b200 as tra
from sparse_attention_video_tra_b200 import build as trabuild
from sparse_attention_video_tra_b200 import synth
import gpu_helpers as gh

pytestmark = pytest.mark.gpu

DISK = oracle.DISK

# (T, H, W, heads, d, gamma, Rt, Bmin, forced tile_w or 0)
CASES = [
    (4, 8, 8, 2, 64, 0.7, 2, 8, 0),
    (3, 7, 9, 2, 128, 0.8, 1, 4, 0),
    (5, 17, 23, 2, 128, 0.8, 3, 8, 0),
    (3, 30, 52, 1, 128, 0.8, 2, 8, 4),
    (4, 19, 21, 2, 64, 0.6, 3, 2, 8),
    (3, 9, 70, 1, 128, 0.9, 2, 3, 32),
    (2, 45, 80, 1, 128, 0.8, 1, 8, 16),
    # the mask kernel's disk-row table covers half-widths up to the frame's cover
    # radius when (S+1)(S+2)/2 <= 12288 entries: 3x155 frames (S = 155) use it,
    # 3x156 frames (S = 156) count the disk row by row
    (2, 3, 155, 1, 64, 0.8, 1, 4, 0),
    (2, 3, 156, 1, 64, 0.8, 1, 4, 0),
]


@pytest.fixture(scope="module", autouse=True)
def built():
    trabuild.build()
    yield


def _ids(c):
    return "x".join(map(str, c[:3])) + f"-d{c[4]}-tw{c[8]}"


def _plan(c, a=1.0, b=0.0, flags=0):
    T, H, W, G, d, gamma, Rt, Bmin, tw = c
    return tra.Plan(T, H, W, G, d, a, b, gamma, Rt, Bmin,
                    flags | tra.TRA_FLAG_DISK | (tra.tra_flag_tile_w(tw) if tw else 0))


@pytest.mark.parametrize("c", CASES, ids=_ids)
def test_disk_radius_and_mask_bit_exact(c):
    T, H, W, G, d, gamma, Rt, Bmin, _ = c
    N = T * H * W
    rng = np.random.default_rng(31 + sum(c[:5]))
    for a, b in ((1.0, 0.0), (1.0, math.log(0.3)), (0.7, 1.5), (0.0, math.log(N / 3.0))):
        plan = _plan(c, a, b)
        i = plan.info
        Hn = rng.uniform(0.0, math.log(N) + 0.3, size=(G, N)).astype(np.float32)
        Hn[:, ::7] = 0.0
        Hn[:, 3::11] = np.float32(50.0)
        mask = plan.new_mask()
        plan.radius_and_mask(gh.to_tile_major(torch.from_numpy(Hn).cuda(), i), mask)
        torch.cuda.synchronize()
        assert plan.status() == 0
        rad, cnt, pairs, _ = plan.mask_views(mask)
        nat = gh.tile_major_index(i)
        rad = rad.cpu().numpy()
        r_gpu = np.zeros((G, N), np.int32)
        r_gpu[:, nat[nat >= 0]] = rad[:, nat >= 0]
        r_o, c_o, _ = oracle.radius(Hn.reshape(-1), G, (T, H, W), a, b, gamma, Rt, Bmin, metric=DISK)
        np.testing.assert_array_equal(r_gpu.reshape(-1), r_o)
        tile_of = np.full(N, -1)
        tile_of[nat[nat >= 0]] = (np.arange(i.N_pad) // 128)[nat >= 0]
        ref_pairs = np.zeros((G, i.n_tiles), np.int64)
        for g in range(G):
            np.add.at(ref_pairs[g], tile_of, c_o.reshape(G, N)[g])
        np.testing.assert_array_equal(pairs.cpu().numpy(), ref_pairs)
        dense = gh.dense_block_mask(plan, mask)
        ref = oracle.block_mask(r_o, G, (T, H, W), gamma, Rt, (i.tile_h, i.tile_w), (i.tile_h, i.tile_w),
                                metric=DISK)
        np.testing.assert_array_equal(dense, ref)
        assert np.all(cnt.cpu().numpy() == (ref.reshape(G, i.n_tiles, -1) > 0).sum(-1))
        plan.close()


@pytest.mark.parametrize("c", CASES, ids=_ids)
def test_disk_attention_matches_oracle(c):
    T, H, W, G, d, gamma, Rt, Bmin, _ = c
    N = T * H * W
    rng = np.random.default_rng(41 + sum(c[:5]))
    plan = _plan(c, 1.0, math.log(0.4))
    i = plan.info
    q, k, v = synth.make_qkv(T, H, W, G, d, 43 + sum(c[:5]), device="cuda", dtype=torch.bfloat16)
    Hn = rng.uniform(0.0, math.log(N), size=(G, N)).astype(np.float32)
    mask = plan.new_mask()
    plan.radius_and_mask(gh.to_tile_major(torch.from_numpy(Hn).cuda(), i), mask)
    qt, kt, vt = (gh.to_tile_major(x, i) for x in (q, k, v))
    out = torch.full((G, i.N_pad, d), float("nan"), device="cuda", dtype=torch.float32)
    plan.attention(qt, kt, vt, mask, out)
    torch.cuda.synchronize()
    assert plan.status() == 0
    o = gh.to_natural(out, i).float().cpu().numpy().reshape(G * N, d)
    r_o, _, _ = oracle.radius(Hn.reshape(-1), G, (T, H, W), 1.0, math.log(0.4), gamma, Rt, Bmin, metric=DISK)
    if G * N > 4000:
        qs = np.sort(rng.choice(G * N, size=400, replace=False))
    else:
        qs = np.arange(G * N)
    ref = oracle.attention(gh.bf16_bits(q), gh.bf16_bits(k), gh.bf16_bits(v), r_o, G, (T, H, W), d, gamma, Rt,
                           queries=qs, metric=DISK)
    gh.check_attention(o[qs], ref)


def test_disk_differs_from_square_and_natural_layout_agrees():
    """The disk keeps fewer pairs than the square at the same radii; the
    natural-layout path gives the tile-major results bit for bit."""
    c = (3, 30, 52, 2, 128, 0.8, 2, 8, 0)
    T, H, W, G, d, gamma, Rt, Bmin, _ = c
    N = T * H * W
    q, k, v = synth.make_qkv(T, H, W, G, d, 77, device="cuda", dtype=torch.bfloat16)
    tm = _plan(c, 1.0, 1.0)
    nat = _plan(c, 1.0, 1.0, tra.TRA_FLAG_NATURAL)
    sq = tra.Plan(T, H, W, G, d, 1.0, 1.0, gamma, Rt, Bmin)
    i = tm.info
    qt, kt, vt = (gh.to_tile_major(x, i) for x in (q, k, v))
    Ht = torch.empty(G, i.N_pad, device="cuda")
    tm.entropy(qt, kt, Ht)
    m_tm, m_sq = tm.new_mask(), sq.new_mask()
    tm.radius_and_mask(Ht, m_tm)
    sq.radius_and_mask(Ht, m_sq)
    o_tm = tm.new_out()
    tm.attention(qt, kt, vt, m_tm, o_tm)
    Hn, m_n, o_n = nat.new_entropy(), nat.new_mask(), nat.new_out()
    nat.entropy(q, k, Hn)
    nat.radius_and_mask(Hn, m_n)
    nat.attention(q, k, v, m_n, o_n)
    torch.cuda.synchronize()
    assert tm.status() == 0 and nat.status() == 0 and sq.status() == 0
    # same budgets: the disk needs a radius at least as large as the square's
    r_d = tm.mask_views(m_tm)[0].cpu().numpy()
    r_s = sq.mask_views(m_sq)[0].cpu().numpy()
    assert np.all(r_d >= r_s) and np.any(r_d > r_s)
    assert torch.equal(gh.to_natural(Ht, i), Hn)
    for a, b in zip(tm.mask_views(m_tm)[:3], nat.mask_views(m_n)[:3]):
        assert torch.equal(a, b)
    assert torch.equal(gh.to_natural(o_tm, i), o_n)
