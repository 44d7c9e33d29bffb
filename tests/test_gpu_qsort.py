"""GPU parity for radius-sorted query groups (TRA_FLAG_QSORT) against the
oracle's query_groups / block_mask_sets.

The rows of each tile-column strip (one tile column of one frame) are
ordered by (radius, strip row), pad rows first; the u-th block of 128 takes
the mask slot of the strip's tile in tile row u.  Checked here:
* radii bit-exact (the same as without the flag, and as the oracle's);
* the group order (mask section `group`) equal to the oracle's;
* every group's key-tile list and full flags equal to the oracle's block
  mask of that query set; the group's retained pairs equal the sum of its
  members' counts;
* attention within max-abs 1e-2 / mean-abs 1e-3 of the fp64 oracle, with the
  Chebyshev square and the disk;
* the natural layout gives the tile-major results bit for bit;
* bf16 output (TRA_FLAG_OUT_BF16) equals the fp32 output rounded to bf16.

Definitions: "Token Radius Attention for Efficient Video Generation"
(gist.science summary), section 2; the grouping is a scheduling choice of
this library and does not change what is computed."""
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

# (T, H, W, heads, d, gamma, Rt, Bmin, forced tile_w or 0); every case has at
# most four tile rows per frame
CASES = [
    (3, 20, 16, 2, 64, 0.7, 2, 8, 8),       # (1,16,8) tiles, ragged rows
    (4, 8, 8, 2, 64, 0.7, 2, 8, 4),         # (1,32,4) tiles, heavy padding
    (3, 19, 21, 2, 128, 0.8, 2, 4, 16),     # (1,8,16) tiles, ragged both ways
    (3, 9, 60, 1, 128, 0.9, 2, 3, 32),      # (1,4,32) tiles
    (2, 45, 80, 1, 128, 0.8, 1, 8, 0),      # 720p frame, (1,16,8) tiles
    (3, 30, 20, 2, 64, 0.8, 2, 8, 16),      # (1,8,16) tiles: four tile rows, odd tile columns
    (3, 48, 24, 2, 64, 0.8, 2, 8, 8),       # (1,16,8) tiles, 3x3 per frame: the odd last frame's slots pair up, one is left alone
]


@pytest.fixture(scope="module", autouse=True)
def built():
    trabuild.build()
    yield


def _ids(c):
    return "x".join(map(str, c[:3])) + f"-d{c[4]}-tw{c[8]}"


def _plan(c, a, b, flags):
    T, H, W, G, d, gamma, Rt, Bmin, tw = c
    return tra.Plan(T, H, W, G, d, a, b, gamma, Rt, Bmin, flags | (tra.tra_flag_tile_w(tw) if tw else 0))


def _radii_natural(plan, mask):
    i = plan.info
    nat = gh.tile_major_index(i)
    rad = plan.mask_views(mask)[0].cpu().numpy()
    r = np.zeros((i.heads, i.N), np.int32)
    r[:, nat[nat >= 0]] = rad[:, nat >= 0]
    return r.reshape(-1)


@pytest.mark.parametrize("metric", [oracle.CHEBYSHEV, oracle.DISK], ids=["square", "disk"])
@pytest.mark.parametrize("c", CASES, ids=_ids)
def test_groups_and_lists_bit_exact(c, metric):
    T, H, W, G, d, gamma, Rt, Bmin, _ = c
    N = T * H * W
    rng = np.random.default_rng(7 + sum(c[:5]))
    extra = tra.TRA_FLAG_DISK if metric == oracle.DISK else 0
    for a, b in ((1.0, 0.0), (1.0, math.log(0.3)), (0.7, 1.5)):
        qs = _plan(c, a, b, tra.TRA_FLAG_QSORT | extra)
        plain = _plan(c, a, b, extra)
        i = qs.info
        Hn = rng.uniform(0.0, math.log(N) + 0.3, size=(G, N)).astype(np.float32)
        Hn[:, ::7] = 0.0
        Ht = gh.to_tile_major(torch.from_numpy(Hn).cuda(), i)
        mq, mp = qs.new_mask(), plain.new_mask()
        qs.radius_and_mask(Ht, mq)
        plain.radius_and_mask(Ht, mp)
        torch.cuda.synchronize()
        assert qs.status() == 0 and plain.status() == 0
        assert torch.equal(qs.mask_views(mq)[0], plain.mask_views(mp)[0])
        r_gpu = _radii_natural(qs, mq)
        r_o, c_o, _ = oracle.radius(Hn.reshape(-1), G, (T, H, W), a, b, gamma, Rt, Bmin, metric=metric)
        np.testing.assert_array_equal(r_gpu, r_o)
        perm, members = oracle.query_groups(r_o, G, (T, H, W), (i.tile_h, i.tile_w))
        np.testing.assert_array_equal(qs.group_view(mq).cpu().numpy().view(np.uint16), perm)
        ref = oracle.block_mask_sets(r_o, G, (T, H, W), gamma, Rt, (i.tile_h, i.tile_w), members, metric=metric)
        np.testing.assert_array_equal(gh.dense_block_mask(qs, mq), ref)
        c_all = c_o.reshape(-1)
        want_pairs = np.where(members >= 0, c_all[np.maximum(members, 0)], 0).sum(axis=1).reshape(G, i.n_tiles)
        np.testing.assert_array_equal(qs.mask_views(mq)[2].cpu().numpy(), want_pairs)
        qs.close()
        plain.close()


@pytest.mark.parametrize("metric", [oracle.CHEBYSHEV, oracle.DISK], ids=["square", "disk"])
@pytest.mark.parametrize("c", CASES, ids=_ids)
def test_attention_matches_oracle(c, metric):
    T, H, W, G, d, gamma, Rt, Bmin, _ = c
    N = T * H * W
    rng = np.random.default_rng(17 + sum(c[:5]))
    extra = tra.TRA_FLAG_DISK if metric == oracle.DISK else 0
    plan = _plan(c, 1.0, math.log(0.4), tra.TRA_FLAG_QSORT | extra)
    i = plan.info
    q, k, v = synth.make_qkv(T, H, W, G, d, 23 + sum(c[:5]), device="cuda", dtype=torch.bfloat16)
    Hn = rng.uniform(0.0, math.log(N), size=(G, N)).astype(np.float32)
    mask = plan.new_mask()
    plan.radius_and_mask(gh.to_tile_major(torch.from_numpy(Hn).cuda(), i), mask)
    qt, kt, vt = (gh.to_tile_major(x, i) for x in (q, k, v))
    out = torch.full((G, i.N_pad, d), float("nan"), device="cuda", dtype=torch.float32)
    plan.attention(qt, kt, vt, mask, out)
    torch.cuda.synchronize()
    assert plan.status() == 0
    o = gh.to_natural(out, i).float().cpu().numpy().reshape(G * N, d)
    r_o, _, _ = oracle.radius(Hn.reshape(-1), G, (T, H, W), 1.0, math.log(0.4), gamma, Rt, Bmin, metric=metric)
    qsel = np.sort(rng.choice(G * N, size=400, replace=False)) if G * N > 4000 else np.arange(G * N)
    ref = oracle.attention(gh.bf16_bits(q), gh.bf16_bits(k), gh.bf16_bits(v), r_o, G, (T, H, W), d, gamma, Rt,
                           queries=qsel, metric=metric)
    gh.check_attention(o[qsel], ref)
    plan.close()


def test_natural_layout_is_bit_identical():
    c = (3, 20, 16, 2, 128, 0.8, 2, 8, 8)
    T, H, W, G, d, gamma, Rt, Bmin, _ = c
    q, k, v = synth.make_qkv(T, H, W, G, d, 91, device="cuda", dtype=torch.bfloat16)
    tm = _plan(c, 1.0, 0.5, tra.TRA_FLAG_QSORT)
    nat = _plan(c, 1.0, 0.5, tra.TRA_FLAG_QSORT | tra.TRA_FLAG_NATURAL)
    i = tm.info
    qt, kt, vt = (gh.to_tile_major(x, i) for x in (q, k, v))
    Ht = torch.empty(G, i.N_pad, device="cuda")
    m_tm, o_tm = tm.new_mask(), tm.new_out()
    tm.entropy(qt, kt, Ht)
    tm.radius_and_mask(Ht, m_tm)
    tm.attention(qt, kt, vt, m_tm, o_tm)
    Hn, m_n, o_n = nat.new_entropy(), nat.new_mask(), nat.new_out()
    nat.entropy(q, k, Hn)
    nat.radius_and_mask(Hn, m_n)
    nat.attention(q, k, v, m_n, o_n)
    torch.cuda.synchronize()
    assert tm.status() == 0 and nat.status() == 0
    assert torch.equal(gh.to_natural(Ht, i), Hn)
    for a, b in zip(tm.mask_views(m_tm)[:3], nat.mask_views(m_n)[:3]):
        assert torch.equal(a, b)
    assert torch.equal(tm.group_view(m_tm), nat.group_view(m_n))
    assert torch.equal(gh.to_natural(o_tm, i), o_n)


@pytest.mark.parametrize("natural", [False, True], ids=["tile-major", "natural"])
@pytest.mark.parametrize("metric", [oracle.CHEBYSHEV, oracle.DISK], ids=["square", "disk"])
@pytest.mark.parametrize("c", [CASES[1], CASES[4], CASES[6]], ids=_ids)
def test_bf16_output_is_the_rounded_fp32_output(c, metric, natural):
    """With query groups each softmax thread writes its own query's row through
    the group map; the bf16 epilogue (TRA_FLAG_OUT_BF16) rounds the same fp32
    value the fp32 epilogue stores, so its rows equal the fp32 rows rounded to
    bf16 (round to nearest even), bit for bit, at every query."""
    T, H, W, G, d, gamma, Rt, Bmin, _ = c
    N = T * H * W
    rng = np.random.default_rng(29 + sum(c[:5]))
    flags = tra.TRA_FLAG_QSORT | (tra.TRA_FLAG_DISK if metric == oracle.DISK else 0) | \
        (tra.TRA_FLAG_NATURAL if natural else 0)
    p32 = _plan(c, 1.0, math.log(0.4), flags)
    p16 = _plan(c, 1.0, math.log(0.4), flags | tra.TRA_FLAG_OUT_BF16)
    i = p32.info
    q, k, v = synth.make_qkv(T, H, W, G, d, 37 + sum(c[:5]), device="cuda", dtype=torch.bfloat16)
    Hn = torch.from_numpy(rng.uniform(0.0, math.log(N), size=(G, N)).astype(np.float32)).cuda()
    if natural:
        qi, ki, vi, Hi = q, k, v, Hn
    else:
        qi, ki, vi = (gh.to_tile_major(x, i) for x in (q, k, v))
        Hi = gh.to_tile_major(Hn, i)
    m32, m16 = p32.new_mask(), p16.new_mask()
    p32.radius_and_mask(Hi, m32)
    p16.radius_and_mask(Hi, m16)
    o32, o16 = p32.new_out(), p16.new_out()
    assert o32.dtype == torch.float32 and o16.dtype == torch.bfloat16
    p32.attention(qi, ki, vi, m32, o32)
    p16.attention(qi, ki, vi, m16, o16)
    torch.cuda.synchronize()
    assert p32.status() == 0 and p16.status() == 0
    for a, b in zip(p32.mask_views(m32)[:3], p16.mask_views(m16)[:3]):
        assert torch.equal(a, b)
    assert torch.equal(p32.group_view(m32), p16.group_view(m16))
    if not natural:
        o32, o16 = gh.to_natural(o32, i), gh.to_natural(o16, i)
    assert torch.equal(o16.view(torch.int16), o32.to(torch.bfloat16).view(torch.int16))
    p32.close()
    p16.close()
