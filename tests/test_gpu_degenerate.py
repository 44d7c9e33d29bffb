"""GPU parity on degenerate grids: a single frame, one-row and one-column
frames, a grid smaller than one 128-token tile, exactly one full tile.

Each case runs the whole path on the GPU -- dense entropy, radius and block
mask, attention -- with the plain layout, radius-sorted query groups
(TRA_FLAG_QSORT), the natural layout (TRA_FLAG_NATURAL) and the Euclidean
disk (TRA_FLAG_DISK), and compares every query with the fp64 oracle:
entropy within 1e-3 relative, radii bit-exact given the GPU's entropies, the
block lists and full bits equal to the oracle's block mask (of the groups'
query sets with TRA_FLAG_QSORT), attention within max-abs 1e-2 / mean-abs 1e-3.

Definitions: "Token Radius Attention for Efficient Video Generation"
(gist.science summary), section 2 ("Entropie-vers-Budget", "Budget-vers-
Rayon", "Noyaux CUDA Fusionnes", "Execution Efficace").  On these grids most
of each (1, th, tw) tile is padding, the temporal reach Rt' = min(Rt, T-1)
is often 0, and a query's neighbourhood is cut by the frame edge in every
direction: the cases where index and clipping mistakes show."""
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

# (T, H, W, heads, d, gamma, Rt, Bmin)
SHAPES = [
    (1, 1, 37, 1, 64, 0.8, 2, 1),       # one frame of one row: two 4x32 tiles, mostly padding
    (1, 5, 7, 2, 128, 0.8, 2, 4),       # 35 tokens: one ragged tile, Rt' = 0
    (2, 3, 1, 1, 64, 0.7, 1, 1),        # a one-column grid of 6 tokens
    (3, 1, 200, 1, 64, 0.8, 2, 8),      # one-row frames, 7 tile columns
    (5, 40, 1, 1, 128, 0.9, 2, 2),      # one-column frames, 2 tile rows
    (1, 16, 8, 1, 64, 0.8, 3, 8),       # exactly one full tile
]
VARIANTS = [(0, "plain"), (tra.TRA_FLAG_QSORT, "qsort"), (tra.TRA_FLAG_NATURAL, "natural"),
            (tra.TRA_FLAG_DISK, "disk")]


@pytest.fixture(scope="module", autouse=True)
def built():
    trabuild.build()
    yield


def _ids(c):
    return "x".join(map(str, c[:3])) + f"-G{c[3]}-d{c[4]}"


@pytest.mark.parametrize("flags,name", VARIANTS, ids=[v[1] for v in VARIANTS])
@pytest.mark.parametrize("c", SHAPES, ids=_ids)
def test_whole_path_on_degenerate_grid(c, flags, name):
    T, H, W, G, d, gamma, Rt, Bmin = c
    N = T * H * W
    metric = oracle.DISK if flags & tra.TRA_FLAG_DISK else oracle.CHEBYSHEV
    natural = bool(flags & tra.TRA_FLAG_NATURAL)
    b = math.log(0.3)
    plan = tra.Plan(T, H, W, G, d, 1.0, b, gamma, Rt, Bmin, flags)
    i = plan.info
    q, k, v = synth.make_qkv(T, H, W, G, d, 31 + sum(c[:5]), device="cuda", dtype=torch.bfloat16)
    if natural:
        qi, ki, vi = q, k, v
        Hg = plan.new_entropy()
    else:
        qi, ki, vi = (gh.to_tile_major(x, i) for x in (q, k, v))
        Hg = torch.empty(G, i.N_pad, device="cuda")
    mask, out = plan.new_mask(), plan.new_out()
    plan.entropy(qi, ki, Hg)
    plan.radius_and_mask(Hg, mask)
    plan.attention(qi, ki, vi, mask, out)
    torch.cuda.synchronize()
    assert plan.status() == 0

    qb, kb, vb = gh.bf16_bits(q), gh.bf16_bits(k), gh.bf16_bits(v)
    Hn = (Hg if natural else gh.to_natural(Hg, i)).cpu().numpy().reshape(-1)
    gh.check_entropy(Hn, oracle.entropy(qb, kb, G, (T, H, W), d))

    r_o, c_o, _ = oracle.radius(Hn, G, (T, H, W), 1.0, b, gamma, Rt, Bmin, metric=metric)
    rad = plan.mask_views(mask)[0].cpu().numpy()
    nat = gh.tile_major_index(i)
    r_gpu = np.zeros((G, N), np.int32)
    r_gpu[:, nat[nat >= 0]] = rad[:, nat >= 0]
    np.testing.assert_array_equal(r_gpu.reshape(-1), r_o)

    tiles = (i.tile_h, i.tile_w)
    if flags & tra.TRA_FLAG_QSORT:
        perm, members = oracle.query_groups(r_o, G, (T, H, W), tiles)
        np.testing.assert_array_equal(plan.group_view(mask).cpu().numpy().view(np.uint16), perm)
        ref = oracle.block_mask_sets(r_o, G, (T, H, W), gamma, Rt, tiles, members, metric=metric)
        want_pairs = np.where(members >= 0, c_o[np.maximum(members, 0)], 0).sum(axis=1).reshape(G, i.n_tiles)
    else:
        ref = oracle.block_mask(r_o, G, (T, H, W), gamma, Rt, tiles, tiles, metric=metric)
        want_pairs = _tile_sums(c_o.reshape(G, N), nat, i)
    np.testing.assert_array_equal(gh.dense_block_mask(plan, mask), ref)
    np.testing.assert_array_equal(plan.mask_views(mask)[2].cpu().numpy(), want_pairs)

    o = (out if natural else gh.to_natural(out, i)).float().cpu().numpy().reshape(G * N, d)
    O_ref = oracle.attention(qb, kb, vb, r_o, G, (T, H, W), d, gamma, Rt, metric=metric)
    gh.check_attention(o, O_ref)
    plan.close()


def _tile_sums(c_nat, nat, info):
    """Retained pairs per query tile: the sum of its valid queries' counts."""
    G = c_nat.shape[0]
    out = np.zeros((G, info.n_tiles), np.int64)
    for p in np.nonzero(nat >= 0)[0]:
        out[:, p // 128] += c_nat[:, nat[p]]
    return out
