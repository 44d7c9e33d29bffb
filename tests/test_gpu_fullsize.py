"""Parity at the workloads' full sizes, through the same launch path the
benchmark times (runner.WorkloadRun: tile-major inputs resident in HBM, b
calibrated to the target retained fraction, entropy -> radius/mask ->
attention).  The oracle computes sampled outputs one by one:

* entropy of sampled queries (dense or every 8th key tile): 1e-3 relative;
* radius of every sampled query from the GPU's own fp32 entropy: bit-exact;
* retained-pair totals of sampled query tiles and their key-tile lists
  (active and full flags): bit-exact;
* attention output rows of sampled queries: max-abs 1e-2, mean-abs 1e-3.

Definitions: "Token Radius Attention for Efficient Video Generation"
(gist.science summary), section 2."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from sparse_attention_video_tra_b200 import build as trabuild
from sparse_attention_video_tra_b200 import synth
from sparse_attention_video_tra_b200.runner import WorkloadRun
import gpu_helpers as gh

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    trabuild.build()
    yield


def _check_run(run: WorkloadRun, heads, n_queries=24, n_tiles=2, seed=0):
    wl, i = run.wl, run.info
    T, H, W, d = wl.T, wl.H, wl.W, wl.d
    N = wl.N
    rng = np.random.default_rng(seed)
    run.run_entropy()
    run.run_mask()
    run.run_attention(0)
    torch.cuda.synchronize()
    assert run.plan.status() == 0
    nat = gh.tile_major_index(i)
    pos_of = np.empty(N, np.int64)
    pos_of[nat[nat >= 0]] = np.nonzero(nat >= 0)[0]
    sel = list(heads)
    G = len(sel)

    def bits_nat(x):                      # [heads, N_pad, d] tile-major -> selected heads, natural, bf16 bits
        return gh.bf16_bits(gh.to_natural(x[sel], i))

    qb, kb, vb = bits_nat(run.q), bits_nat(run.k), bits_nat(run.v[0])
    out = gh.to_natural(run.out[sel], i).float().cpu().numpy().reshape(G * N, d)
    Hg = gh.to_natural(run.H[sel], i).cpu().numpy().reshape(G * N)
    rad = run.plan.mask_views(run.mask)[0][sel].cpu().numpy()
    r_nat = np.zeros((G, N), np.int32)
    r_nat[:, nat[nat >= 0]] = rad[:, nat >= 0]
    r_nat = r_nat.reshape(-1)

    queries = np.sort(rng.choice(G * N, size=n_queries, replace=False))
    # entropy (dense or subsampled over the library's key tiles)
    Href = oracle.entropy(qb, kb, G, (T, H, W), d, key_stride=wl.key_stride, ktile=(i.tile_h, i.tile_w),
                          queries=queries)
    gh.check_entropy(Hg[queries], Href)
    # radius from the GPU's fp32 entropies: bit-exact
    r_ref, c_ref, _ = oracle.radius(Hg[queries], G, (T, H, W), wl.a, run.b, wl.gamma, wl.Rt, wl.Bmin,
                                    queries=queries)
    np.testing.assert_array_equal(r_nat[queries], r_ref)
    # attention rows
    Oref = oracle.attention(qb, kb, vb, r_nat, G, (T, H, W), d, wl.gamma, wl.Rt, queries=queries)
    gh.check_attention(out[queries], Oref)
    # block-mask rows and retained pairs of sampled query tiles
    _, cnt, pairs, lst = run.plan.mask_views(run.mask)
    for t in rng.choice(i.n_tiles, size=n_tiles, replace=False):
        for gi, g in enumerate(sel):
            row = oracle.block_mask(r_nat, G, (T, H, W), wl.gamma, wl.Rt, (i.tile_h, i.tile_w),
                                    (i.tile_h, i.tile_w), qtiles=[gi * i.n_tiles + int(t)])[0]
            n = int(cnt[g, t])
            e = lst[g, t, :n].cpu().numpy().view(np.uint16).astype(np.int64)
            dense = np.zeros(i.n_tiles, np.uint8)
            dense[e & 0x7FFF] = np.where(e & 0x8000, 3, 1)
            np.testing.assert_array_equal(dense, row)
            members = nat[t * 128:(t + 1) * 128]
            members = members[members >= 0] + gi * N
            _, c_mem, _ = oracle.radius(Hg[members], G, (T, H, W), wl.a, run.b, wl.gamma, wl.Rt, wl.Bmin,
                                        queries=members)
            assert int(pairs[g, t]) == int(c_mem.sum())


def test_wan720_full_size_bench_configuration():
    """Wan-14B-720p: 21x45x80, 40 heads, d=128, dense warm-up entropy."""
    run = WorkloadRun(synth.WORKLOADS["wan720"], calls=1)
    assert abs(run.retained_fraction_now() - 0.15) < 0.01
    _check_run(run, heads=(0, 39), n_queries=24, n_tiles=2, seed=1)


def test_wan480_full_size():
    run = WorkloadRun(synth.WORKLOADS["wan480"], calls=1)
    _check_run(run, heads=(3, 11), n_queries=32, n_tiles=3, seed=2)


def test_hunyuan720_full_size_subsampled_entropy():
    """HunyuanVideo-720p: 33x45x80, 24 heads, entropy from every 8th key tile."""
    run = WorkloadRun(synth.WORKLOADS["hunyuan720"], calls=1)
    _check_run(run, heads=(5,), n_queries=24, n_tiles=2, seed=3)


def test_len4x_full_size():
    """4x length: 132x45x80 (475,200 tokens), 24 heads, gamma 0.7, Rt 16."""
    run = WorkloadRun(synth.WORKLOADS["len4x"], calls=1)
    _check_run(run, heads=(0, 23), n_queries=12, n_tiles=1, seed=4)


def test_tiny_workload_complete():
    """The tiny oracle case in full: every output, radius and list entry."""
    run = WorkloadRun(synth.WORKLOADS["tiny"], calls=1)
    _check_run(run, heads=(0, 1), n_queries=2 * 256, n_tiles=4, seed=5)
