"""Natural token order (TRA_FLAG_NATURAL) against the tile-major path.

With the flag the kernels load each (1, th, tw) tile straight from
[heads][T][H][W][d] through a 4-D TMA box, which lands in the same
shared-memory rows as a tile-major load, and write entropies and outputs
back to their natural rows.  The arithmetic is unchanged, so every result
must equal the tile-major path's bit for bit: entropies, the whole mask
buffer (radii, counts, retained pairs, lists) and the attention output.
The tile-major path itself is checked against the oracle elsewhere; one
case here is also checked against the oracle directly on sampled rows.

Layouts: "Token Radius Attention for Efficient Video Generation"
(gist.science summary), section 2, "Disposition Tile-Major"."""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_video_tra_b200 as tra
from sparse_attention_video_tra_b200 import build as trabuild
from sparse_attention_video_tra_b200 import synth
import gpu_helpers as gh

pytestmark = pytest.mark.gpu

# (T, H, W, heads, d, gamma, Rt, Bmin, forced tile_w or 0)
CASES = [
    (4, 8, 8, 2, 64, 0.7, 2, 8, 0),        # (1,16,8) tiles, half padding in h
    (4, 8, 8, 2, 64, 0.7, 2, 8, 16),       # (1,8,16) tiles, half padding in w
    (3, 7, 9, 2, 128, 0.8, 1, 4, 0),       # one ragged tile per frame
    (5, 17, 23, 2, 128, 0.8, 3, 8, 0),     # ragged both ways
    (3, 30, 52, 1, 128, 0.8, 2, 8, 4),     # (1,32,4) tiles
    (4, 19, 21, 2, 64, 0.6, 3, 2, 8),      # (1,16,8) tiles
    (3, 9, 70, 1, 128, 0.9, 2, 3, 32),     # (1,4,32) tiles
]


@pytest.fixture(scope="module", autouse=True)
def built():
    trabuild.build()
    yield


def _ids(c):
    return "x".join(map(str, c[:3])) + f"-d{c[4]}-tw{c[8]}"


def _plans(c, b=0.0, extra=0):
    T, H, W, G, d, gamma, Rt, Bmin, tw = c
    f = extra | (tra.tra_flag_tile_w(tw) if tw else 0)
    return (tra.Plan(T, H, W, G, d, 1.0, b, gamma, Rt, Bmin, f),
            tra.Plan(T, H, W, G, d, 1.0, b, gamma, Rt, Bmin, f | tra.TRA_FLAG_NATURAL))


def _run(c, stride=1, b=0.0, extra=0, seed=11):
    T, H, W, G, d = c[:5]
    tm, nat = _plans(c, b, extra)
    i = tm.info
    q, k, v = synth.make_qkv(T, H, W, G, d, seed, device="cuda", dtype=torch.bfloat16)
    # tile-major path (inputs permuted on the host side of the test)
    qt, kt, vt = (gh.to_tile_major(x, i) for x in (q, k, v))
    Ht = torch.empty(G, i.N_pad, device="cuda")
    mt = tm.new_mask()
    ot = tm.new_out()
    tm.entropy(qt, kt, Ht, stride)
    tm.radius_and_mask(Ht, mt)
    tm.attention(qt, kt, vt, mt, ot)
    # natural path straight from the frame-major tensors
    Hn = nat.new_entropy()
    mn = nat.new_mask()
    on = nat.new_out()
    nat.entropy(q, k, Hn, stride)
    nat.radius_and_mask(Hn, mn)
    nat.attention(q, k, v, mn, on)
    torch.cuda.synchronize()
    assert tm.status() == 0 and nat.status() == 0
    return tm, nat, (q, k, v), (Ht, mt, ot), (Hn, mn, on)


def _same_mask(plan, a, b):
    ra, ca, pa, la = plan.mask_views(a)
    rb, cb, pb, lb = plan.mask_views(b)
    assert torch.equal(ra, rb)
    assert torch.equal(ca, cb)
    assert torch.equal(pa, pb)
    cnt = ca.cpu().numpy()
    la, lb = la.cpu().numpy(), lb.cpu().numpy()
    for g in range(cnt.shape[0]):
        for t in range(cnt.shape[1]):
            n = int(cnt[g, t])
            np.testing.assert_array_equal(la[g, t, :n], lb[g, t, :n])


@pytest.mark.parametrize("c", CASES, ids=_ids)
def test_natural_equals_tile_major_bitwise(c):
    tm, nat, _, (Ht, mt, ot), (Hn, mn, on) = _run(c)
    i = tm.info
    assert torch.equal(gh.to_natural(Ht, i), Hn)
    _same_mask(tm, mt, mn)
    assert torch.equal(gh.to_natural(ot, i), on)


@pytest.mark.parametrize("c", [CASES[2], CASES[5]], ids=_ids)
def test_natural_subsampled_entropy_and_bf16_output(c):
    tm, nat, _, (Ht, mt, ot), (Hn, mn, on) = _run(c, stride=3, extra=tra.TRA_FLAG_OUT_BF16, seed=12)
    i = tm.info
    assert on.dtype == torch.bfloat16
    assert torch.equal(gh.to_natural(Ht, i), Hn)
    _same_mask(tm, mt, mn)
    assert torch.equal(gh.to_natural(ot, i), on)


def test_natural_against_oracle():
    """Natural layout on a 720p frame pair, sampled rows against the oracle."""
    c = (2, 45, 80, 1, 128, 0.8, 1, 8, 16)
    T, H, W, G, d, gamma, Rt = c[:7]
    tm, nat, (q, k, v), _, (Hn, mn, on) = _run(c, b=2.0, seed=13)
    N = T * H * W
    rng = np.random.default_rng(3)
    qs = np.sort(rng.choice(N, size=48, replace=False))
    qb, kb, vb = gh.bf16_bits(q), gh.bf16_bits(k), gh.bf16_bits(v)
    Href = oracle.entropy(qb, kb, G, (T, H, W), d, queries=qs)
    gh.check_entropy(Hn.cpu().numpy().reshape(-1)[qs], Href)
    r_nat = np.zeros(N, np.int32)
    nat_idx = gh.tile_major_index(nat.info)
    rad = nat.mask_views(mn)[0][0].cpu().numpy()
    r_nat[nat_idx[nat_idx >= 0]] = rad[nat_idx >= 0]
    Oref = oracle.attention(qb, kb, vb, r_nat, G, (T, H, W), d, gamma, Rt, queries=qs)
    gh.check_attention(on.float().cpu().numpy().reshape(N, d)[qs], Oref)


def test_natural_rejects_tile_major_sized_buffers():
    c = CASES[1]
    tm, nat = _plans(c)
    q = tm.new_tile_major()
    with pytest.raises(ValueError):
        nat.attention(q, q, q, nat.new_mask(), nat.new_out())
