"""Robustness of the device path: a corrupted mask buffer is detected and
reported, never dereferenced out of range; and every result is deterministic
(two runs are bit-identical), which the exact-mask design requires of the
radii and lists and which holds for entropies and outputs as well.

The mask buffer is caller memory shared across calls ("Reutilisation
Inter-Etapes" in "Token Radius Attention for Efficient Video Generation",
gist.science summary, section 2), so tra_attention validates what it reads:
tile counts within [0, list_cap] and listed tiles within the reach of the
query tile pair."""
import numpy as np
import pytest
import torch

import sparse_attention_video_tra_b200 as tra
from sparse_attention_video_tra_b200 import build as trabuild
from sparse_attention_video_tra_b200 import synth
import gpu_helpers as gh

pytestmark = pytest.mark.gpu

C = (5, 17, 23, 2, 128, 0.8, 3, 8)


@pytest.fixture(scope="module", autouse=True)
def built():
    trabuild.build()
    yield


def _setup(seed=3):
    T, H, W, G, d, gamma, Rt, Bmin = C
    plan = tra.Plan(T, H, W, G, d, 1.0, 0.5, gamma, Rt, Bmin)
    i = plan.info
    q, k, v = synth.make_qkv(T, H, W, G, d, seed, device="cuda", dtype=torch.bfloat16)
    qt, kt, vt = (gh.to_tile_major(x, i) for x in (q, k, v))
    Ht = torch.empty(G, i.N_pad, device="cuda")
    plan.entropy(qt, kt, Ht)
    mask = plan.new_mask()
    plan.radius_and_mask(Ht, mask)
    torch.cuda.synchronize()
    assert plan.status() == 0
    return plan, (qt, kt, vt), Ht, mask


def test_corrupted_tile_count_is_reported_not_followed():
    plan, (qt, kt, vt), _, mask = _setup()
    bad = mask.clone()
    cnt = plan.mask_views(bad)[1]
    cnt[0, 0] = plan.info.list_cap + 7
    cnt[1, 3] = -2
    out = plan.new_out()
    plan.attention(qt, kt, vt, bad, out)
    torch.cuda.synchronize()
    assert plan.status() == 6                       # TRA_ERR_DEVICE_CHECK
    # the context and the valid mask still work
    plan.attention(qt, kt, vt, mask, out)
    torch.cuda.synchronize()
    assert plan.status() == 0
    assert torch.isfinite(gh.to_natural(out, plan.info)).all()


def test_unreachable_list_entry_is_reported_and_skipped():
    plan, (qt, kt, vt), _, mask = _setup()
    bad = mask.clone()
    lst = plan.mask_views(bad)[3]
    lst[0, 0, 0] = 0x7FFE                           # a tile id no query of tile 0 can reach
    out = plan.new_out()
    plan.attention(qt, kt, vt, bad, out)
    torch.cuda.synchronize()
    assert plan.status() == 6


def test_list_entry_beyond_its_own_tiles_reach_is_reported():
    """A listed key tile Rt' + 1 frames from the query tile that lists it is
    still inside the range of key tiles the CTA's pair of query tiles could
    reach together, so it must be caught by the per-list frame check (the
    half-width table has no row for that frame distance)."""
    plan, (qt, kt, vt), _, mask = _setup()
    i = plan.info
    tpf = i.n_tiles_h * i.n_tiles_w
    assert i.rt_eff + 1 < i.T
    bad = mask.clone()
    lst = plan.mask_views(bad)[3]
    lst[0, 0, 0] = (i.rt_eff + 1) * tpf              # frame Rt'+1; tile 0 sits in frame 0
    out = plan.new_out()
    plan.attention(qt, kt, vt, bad, out)
    torch.cuda.synchronize()
    assert plan.status() == 6
    plan.attention(qt, kt, vt, mask, out)
    torch.cuda.synchronize()
    assert plan.status() == 0


def test_group_entry_past_the_strip_is_reported():
    """With radius-sorted groups each slot names a strip row; a row past the
    strip (128 * n_tiles_h or more) is recorded, never followed."""
    T, H, W, G, d, gamma, Rt, Bmin = C
    plan = tra.Plan(T, H, W, G, d, 1.0, 0.5, gamma, Rt, Bmin, tra.TRA_FLAG_QSORT | tra.tra_flag_tile_w(8))
    i = plan.info
    q, k, v = synth.make_qkv(T, H, W, G, d, 5, device="cuda", dtype=torch.bfloat16)
    qt, kt, vt = (gh.to_tile_major(x, i) for x in (q, k, v))
    Ht = torch.empty(G, i.N_pad, device="cuda")
    plan.entropy(qt, kt, Ht)
    mask = plan.new_mask()
    plan.radius_and_mask(Ht, mask)
    torch.cuda.synchronize()
    assert plan.status() == 0
    bad = mask.clone()
    plan.group_view(bad)[1, 2, 5] = 0x7FFF
    out = plan.new_out()
    plan.attention(qt, kt, vt, bad, out)
    torch.cuda.synchronize()
    assert plan.status() == 6
    plan.attention(qt, kt, vt, mask, out)
    torch.cuda.synchronize()
    assert plan.status() == 0


def test_results_are_bit_identical_across_runs():
    plan, (qt, kt, vt), Ht, mask = _setup(seed=9)
    i = plan.info
    H2 = torch.empty_like(Ht)
    plan.entropy(qt, kt, H2)
    mask2 = plan.new_mask()
    plan.radius_and_mask(H2, mask2)
    o1, o2 = plan.new_out(), plan.new_out()
    plan.attention(qt, kt, vt, mask, o1)
    plan.attention(qt, kt, vt, mask2, o2)
    torch.cuda.synchronize()
    assert plan.status() == 0
    nat = torch.from_numpy(gh.tile_major_index(i) >= 0).cuda()
    assert torch.equal(Ht[:, nat], H2[:, nat])
    a, b = plan.mask_views(mask), plan.mask_views(mask2)
    for x, y in zip(a[:3], b[:3]):
        assert torch.equal(x, y)
    cnt = a[1].cpu().numpy()
    la, lb = a[3].cpu().numpy(), b[3].cpu().numpy()
    for g in range(i.heads):
        for t in range(i.n_tiles):
            n = int(cnt[g, t])
            np.testing.assert_array_equal(la[g, t, :n], lb[g, t, :n])
    assert torch.equal(o1[:, nat], o2[:, nat])
