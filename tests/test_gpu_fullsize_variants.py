"""Full-size parity of the plan variants at the Wan-720p bench shape
(21x45x80, 40 heads, d=128, 15 % of pairs retained), through the same
resident-input path the benchmark times:

* the Euclidean disk (TRA_FLAG_DISK) against the oracle's metric 1 on
  sampled queries and query tiles: radii and block-mask rows bit-exact,
  attention within max-abs 1e-2 / mean-abs 1e-3;
* the natural token order (TRA_FLAG_NATURAL) against the tile-major path:
  entropies, mask buffer and outputs bit for bit.

Definitions: "Token Radius Attention for Efficient Video Generation"
(gist.science summary), section 2; the disk is Intuition II's circular
neighbourhood."""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_video_tra_b200 as tra
from sparse_attention_video_tra_b200 import build as trabuild
from sparse_attention_video_tra_b200 import synth
from sparse_attention_video_tra_b200.runner import WorkloadRun
import gpu_helpers as gh

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def run():
    trabuild.build()
    r = WorkloadRun(synth.WORKLOADS["wan720"], calls=1)
    r.run_entropy()
    r.run_mask()
    r.run_attention(0)
    torch.cuda.synchronize()
    assert r.plan.status() == 0
    yield r


def _plan(run, flags):
    wl = run.wl
    return tra.Plan(wl.T, wl.H, wl.W, wl.heads, wl.d, wl.a, run.b, wl.gamma, wl.Rt, wl.Bmin, flags)


def test_wan720_full_size_disk(run):
    wl, i = run.wl, run.info
    T, H, W, d, N = wl.T, wl.H, wl.W, wl.d, wl.N
    plan = _plan(run, tra.TRA_FLAG_DISK)
    mask, out = plan.new_mask(), plan.new_out()
    plan.radius_and_mask(run.H, mask)
    plan.attention(run.q, run.k, run.v[0], mask, out)
    torch.cuda.synchronize()
    assert plan.status() == 0
    rng = np.random.default_rng(11)
    sel = [0, wl.heads - 1]
    G = len(sel)
    nat = gh.tile_major_index(i)
    bits = lambda x: gh.bf16_bits(gh.to_natural(x[sel], i))     # noqa: E731
    qb, kb, vb = bits(run.q), bits(run.k), bits(run.v[0])
    o = gh.to_natural(out[sel], i).float().cpu().numpy().reshape(G * N, d)
    Hg = gh.to_natural(run.H[sel], i).cpu().numpy().reshape(G * N)
    rad, cnt, pairs, lst = plan.mask_views(mask)
    r_nat = np.zeros((G, N), np.int32)
    r_nat[:, nat[nat >= 0]] = rad[sel].cpu().numpy()[:, nat >= 0]
    r_nat = r_nat.reshape(-1)
    queries = np.sort(rng.choice(G * N, size=24, replace=False))
    r_ref, _, _ = oracle.radius(Hg[queries], G, (T, H, W), wl.a, run.b, wl.gamma, wl.Rt, wl.Bmin,
                                queries=queries, metric=oracle.DISK)
    np.testing.assert_array_equal(r_nat[queries], r_ref)
    Oref = oracle.attention(qb, kb, vb, r_nat, G, (T, H, W), d, wl.gamma, wl.Rt, queries=queries,
                            metric=oracle.DISK)
    gh.check_attention(o[queries], Oref)
    for t in rng.choice(i.n_tiles, size=2, replace=False):
        for gi, g in enumerate(sel):
            row = oracle.block_mask(r_nat, G, (T, H, W), wl.gamma, wl.Rt, (i.tile_h, i.tile_w),
                                    (i.tile_h, i.tile_w), qtiles=[gi * i.n_tiles + int(t)], metric=oracle.DISK)[0]
            n = int(cnt[g, t])
            e = lst[g, t, :n].cpu().numpy().view(np.uint16).astype(np.int64)
            dense = np.zeros(i.n_tiles, np.uint8)
            dense[e & 0x7FFF] = np.where(e & 0x8000, 3, 1)
            np.testing.assert_array_equal(dense, row)
            members = nat[t * 128:(t + 1) * 128]
            members = members[members >= 0] + gi * N
            _, c_mem, _ = oracle.radius(Hg[members], G, (T, H, W), wl.a, run.b, wl.gamma, wl.Rt, wl.Bmin,
                                        queries=members, metric=oracle.DISK)
            assert int(pairs[g, t]) == int(c_mem.sum())
    plan.close()


def test_wan720_full_size_natural_layout_is_bit_identical(run):
    wl, i = run.wl, run.info
    plan = _plan(run, tra.TRA_FLAG_NATURAL)
    q, k, v = (gh.to_natural(x, i).contiguous() for x in (run.q, run.k, run.v[0]))
    Hn, mask, out = plan.new_entropy(), plan.new_mask(), plan.new_out()
    plan.entropy(q, k, Hn, wl.key_stride)
    plan.radius_and_mask(Hn, mask)
    plan.attention(q, k, v, mask, out)
    torch.cuda.synchronize()
    assert plan.status() == 0
    assert torch.equal(gh.to_natural(run.H, i), Hn)
    a, b = run.plan.mask_views(run.mask), plan.mask_views(mask)
    for x, y in zip(a[:3], b[:3]):                    # radii, tile counts, pair sums
        assert torch.equal(x, y)
    listed = torch.arange(i.list_cap, device=a[1].device).view(1, 1, -1) < a[1].unsqueeze(-1)
    assert torch.equal(a[3][listed], b[3][listed])    # every listed entry, full flags included
    assert torch.equal(gh.to_natural(run.out, i), out)
    plan.close()


def test_wan720_full_size_qsort(run):
    """Radius-sorted query groups (TRA_FLAG_QSORT, the benchmark's default at
    this shape): radii as without the flag, the group order and sampled group
    lists equal to the oracle's, sampled outputs within tolerance."""
    wl, i = run.wl, run.info
    T, H, W, d, N = wl.T, wl.H, wl.W, wl.d, wl.N
    plan = _plan(run, tra.TRA_FLAG_QSORT)
    mask, out = plan.new_mask(), plan.new_out()
    plan.radius_and_mask(run.H, mask)
    plan.attention(run.q, run.k, run.v[0], mask, out)
    torch.cuda.synchronize()
    assert plan.status() == 0
    rad, cnt, pairs, lst = plan.mask_views(mask)
    assert torch.equal(rad, run.plan.mask_views(run.mask)[0])
    rng = np.random.default_rng(13)
    sel = [0, wl.heads - 1]
    G = len(sel)
    nat = gh.tile_major_index(i)
    r_nat = np.zeros((G, N), np.int32)
    r_nat[:, nat[nat >= 0]] = rad[sel].cpu().numpy()[:, nat >= 0]
    r_nat = r_nat.reshape(-1)
    perm, members = oracle.query_groups(r_nat, G, (T, H, W), (i.tile_h, i.tile_w))
    np.testing.assert_array_equal(plan.group_view(mask)[sel].cpu().numpy().view(np.uint16), perm)
    Hg = gh.to_natural(run.H[sel], i).cpu().numpy().reshape(G * N)
    for t in rng.choice(i.n_tiles, size=3, replace=False):
        for gi, g in enumerate(sel):
            mem = members[gi * i.n_tiles + int(t)][None]
            row = oracle.block_mask_sets(r_nat, G, (T, H, W), wl.gamma, wl.Rt, (i.tile_h, i.tile_w), mem)[0]
            n = int(cnt[g, t])
            e = lst[g, t, :n].cpu().numpy().view(np.uint16).astype(np.int64)
            dense = np.zeros(i.n_tiles, np.uint8)
            dense[e & 0x7FFF] = np.where(e & 0x8000, 3, 1)
            np.testing.assert_array_equal(dense, row)
            q = mem[0][mem[0] >= 0]
            _, c_mem, _ = oracle.radius(Hg[q], G, (T, H, W), wl.a, run.b, wl.gamma, wl.Rt, wl.Bmin, queries=q)
            assert int(pairs[g, t]) == int(c_mem.sum())
    bits = lambda x: gh.bf16_bits(gh.to_natural(x[sel], i))     # noqa: E731
    qb, kb, vb = bits(run.q), bits(run.k), bits(run.v[0])
    o = gh.to_natural(out[sel], i).float().cpu().numpy().reshape(G * N, d)
    queries = np.sort(rng.choice(G * N, size=24, replace=False))
    Oref = oracle.attention(qb, kb, vb, r_nat, G, (T, H, W), d, wl.gamma, wl.Rt, queries=queries)
    gh.check_attention(o[queries], Oref)
    plan.close()


@pytest.mark.parametrize("metric", [oracle.CHEBYSHEV, oracle.DISK], ids=["square", "disk"])
def test_wan720_every_cta_of_the_grouped_launch(run, metric):
    """The benchmark's own configuration (TRA_FLAG_QSORT: radius-sorted
    tile-column strips) at full size, covering every CTA of the attention
    launch: each CTA takes slot s of frames 2f and 2f + 1, or two adjacent
    slots of the odd last frame 20, and one query of each of its slots is checked against the
    oracle -- radius bit-exact, output row within max-abs 1e-2 / mean-abs
    1e-3 -- for two heads, with the Chebyshev square and with the disk.  The
    group order equals the oracle's everywhere, and one group list per frame
    pair equals the oracle's block mask of that group's members."""
    wl, i = run.wl, run.info
    T, H, W, d, N = wl.T, wl.H, wl.W, wl.d, wl.N
    disk = metric == oracle.DISK
    plan = _plan(run, tra.TRA_FLAG_QSORT | (tra.TRA_FLAG_DISK if disk else 0))
    mask, out = plan.new_mask(), plan.new_out()
    plan.radius_and_mask(run.H, mask)
    plan.attention(run.q, run.k, run.v[0], mask, out)
    torch.cuda.synchronize()
    assert plan.status() == 0
    rng = np.random.default_rng(29 + metric)
    sel = [0, wl.heads - 1]
    G = len(sel)
    tpf = i.n_tiles_h * i.n_tiles_w
    nat = gh.tile_major_index(i)
    rad, cnt, pairs, lst = plan.mask_views(mask)
    r_nat = np.zeros((G, N), np.int32)
    r_nat[:, nat[nat >= 0]] = rad[sel].cpu().numpy()[:, nat >= 0]
    r_nat = r_nat.reshape(-1)
    Hg = gh.to_natural(run.H[sel], i).cpu().numpy().reshape(G * N)
    perm, members = oracle.query_groups(r_nat, G, (T, H, W), (i.tile_h, i.tile_w))
    np.testing.assert_array_equal(plan.group_view(mask)[sel].cpu().numpy().view(np.uint16), perm)
    # the launch: CTA p < (T // 2) * tpf takes slot s = p % tpf of frames 2f
    # and 2f + 1; the rest take slots 2k, 2k + 1 of the odd last frame
    slots = []
    paired = T // 2 * tpf
    n_cta = paired + (T % 2) * ((tpf + 1) // 2)
    for p in range(n_cta):
        if p < paired:
            qa = 2 * (p // tpf) * tpf + p % tpf
            qb = qa + tpf
        else:
            qa = (T - 1) * tpf + 2 * (p - paired)
            qb = qa + 1
        slots += [qa] + ([qb] if qb < i.n_tiles else [])
    assert sorted(slots) == list(range(i.n_tiles))         # every slot in exactly one CTA
    queries = []
    for gi in range(G):
        for a in slots:
            m = members[gi * i.n_tiles + a]
            queries.append(int(rng.choice(m[m >= 0])))
    queries = np.array(sorted(set(queries)))
    assert len(queries) >= 0.99 * G * i.n_tiles          # one query per slot of every CTA
    r_ref, _, _ = oracle.radius(Hg[queries], G, (T, H, W), wl.a, run.b, wl.gamma, wl.Rt, wl.Bmin,
                                queries=queries, metric=metric)
    np.testing.assert_array_equal(r_nat[queries], r_ref)
    bits = lambda x: gh.bf16_bits(gh.to_natural(x[sel], i))     # noqa: E731
    qb, kb, vb = bits(run.q), bits(run.k), bits(run.v[0])
    o = gh.to_natural(out[sel], i).float().cpu().numpy().reshape(G * N, d)
    Oref = oracle.attention(qb, kb, vb, r_nat, G, (T, H, W), d, wl.gamma, wl.Rt, queries=queries, metric=metric)
    gh.check_attention(o[queries], Oref)
    # one group list per frame pair and head
    for f in range(0, T, 2):
        a = f * tpf + int(rng.integers(tpf))
        for gi, g in enumerate(sel):
            mem = members[gi * i.n_tiles + a][None]
            row = oracle.block_mask_sets(r_nat, G, (T, H, W), wl.gamma, wl.Rt, (i.tile_h, i.tile_w), mem,
                                         metric=metric)[0]
            n = int(cnt[g, a])
            e = lst[g, a, :n].cpu().numpy().view(np.uint16).astype(np.int64)
            dense = np.zeros(i.n_tiles, np.uint8)
            dense[e & 0x7FFF] = np.where(e & 0x8000, 3, 1)
            np.testing.assert_array_equal(dense, row)
            q = mem[0][mem[0] >= 0]
            _, c_mem, _ = oracle.radius(Hg[q], G, (T, H, W), wl.a, run.b, wl.gamma, wl.Rt, wl.Bmin, queries=q,
                                        metric=metric)
            assert int(pairs[g, a]) == int(c_mem.sum())
    plan.close()
