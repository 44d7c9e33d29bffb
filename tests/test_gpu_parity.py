"""GPU parity of every kernel against the fp64 oracle, through the C ABI, at
sizes the oracle finishes in seconds that still span several tiles, ragged
(padded) tile edges, both head dims and all four tile widths.

Definitions: "Token Radius Attention for Efficient Video Generation"
(gist.science summary), section 2 (entropy -> budget -> radius -> mask ->
block-sparse attention)."""
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

# (T, H, W, heads, d, gamma, Rt, Bmin, forced tile_w or 0)
CASES = [
    (4, 8, 8, 2, 64, 0.7, 2, 8, 0),        # tiny workload shape: (1,16,8) tiles, half padding in h
    (4, 8, 8, 2, 64, 0.7, 2, 8, 16),       # the same in (1,8,16) tiles, half padding in w
    (3, 7, 9, 2, 128, 0.8, 1, 4, 0),       # one ragged tile per frame
    (5, 17, 23, 2, 128, 0.8, 3, 8, 0),     # several tiles, ragged both ways
    (3, 30, 52, 1, 128, 0.8, 2, 8, 4),     # Wan-480p frame, (1,32,4) tiles
    (4, 19, 21, 2, 64, 0.6, 3, 2, 8),      # (1,16,8) tiles
    (3, 9, 70, 1, 128, 0.9, 2, 3, 32),     # (1,4,32) tiles
    (2, 45, 80, 1, 128, 0.8, 1, 8, 0),     # 720p frame, (1,16,8) tiles
    (2, 45, 80, 1, 128, 0.8, 1, 8, 16),    # 720p frame, (1,8,16) tiles
]


@pytest.fixture(scope="module", autouse=True)
def built():
    trabuild.build()
    yield


def _ids(c):
    return "x".join(map(str, c[:3])) + f"-d{c[4]}-tw{c[8]}"


def _plan(c, a=1.0, b=0.0, flags=0):
    T, H, W, G, d, gamma, Rt, Bmin, tw = c
    return tra.Plan(T, H, W, G, d, a, b, gamma, Rt, Bmin, flags | (tra.tra_flag_tile_w(tw) if tw else 0))


def _qkv(c, seed):
    T, H, W, G, d = c[:5]
    return synth.make_qkv(T, H, W, G, d, seed, device="cuda", dtype=torch.bfloat16)


@pytest.mark.parametrize("c", CASES, ids=_ids)
def test_permute_round_trip(c):
    plan = _plan(c)
    i = plan.info
    x = torch.randn(i.heads, i.N, i.d, device="cuda").to(torch.bfloat16)
    tm = torch.full((i.heads, i.N_pad, i.d), float("nan"), device="cuda", dtype=torch.bfloat16)
    plan.permute(x, tm, True)
    back = torch.empty_like(x)
    plan.permute(tm, back, False)
    torch.cuda.synchronize()
    assert torch.equal(back.view(torch.int16), x.view(torch.int16))
    ref = gh.to_tile_major(x, i)
    assert torch.equal(tm.view(torch.int16), ref.view(torch.int16))      # pads are zeros, rows in place
    xf = torch.randn(i.heads, i.N, i.d, device="cuda")
    tf = torch.full((i.heads, i.N_pad, i.d), float("nan"), device="cuda")
    plan.permute(xf, tf, True)
    bf = torch.empty_like(xf)
    plan.permute(tf, bf, False)
    torch.cuda.synchronize()
    assert torch.equal(bf, xf) and torch.equal(tf, gh.to_tile_major(xf, i))
    assert plan.status() == 0


@pytest.mark.parametrize("c", CASES, ids=_ids)
def test_radius_and_mask_bit_exact(c):
    T, H, W, G, d, gamma, Rt, Bmin, _ = c
    N = T * H * W
    rng = np.random.default_rng(sum(c[:5]))
    for a, b in ((1.0, 0.0), (1.0, math.log(0.3)), (0.7, 1.5), (0.0, math.log(N / 3.0))):
        plan = _plan(c, a, b)
        i = plan.info
        Hn = rng.uniform(0.0, math.log(N) + 0.3, size=(G, N)).astype(np.float32)
        Hn[:, ::7] = 0.0                     # budget at Bmin
        Hn[:, 3::11] = np.float32(50.0)      # budget clamped at N
        Ht = gh.to_tile_major(torch.from_numpy(Hn).cuda(), i)
        mask = plan.new_mask()
        plan.radius_and_mask(Ht, mask)
        torch.cuda.synchronize()
        assert plan.status() == 0
        rad, cnt, pairs, _ = plan.mask_views(mask)
        nat = gh.tile_major_index(i)
        rad = rad.cpu().numpy()
        assert np.all(rad[:, nat < 0] == -1)
        r_gpu = np.zeros((G, N), np.int32)
        r_gpu[:, nat[nat >= 0]] = rad[:, nat >= 0]
        r_o, c_o, _ = oracle.radius(Hn.reshape(-1), G, (T, H, W), a, b, gamma, Rt, Bmin)
        np.testing.assert_array_equal(r_gpu.reshape(-1), r_o)
        # retained pairs per tile
        tile_of = np.full(N, -1)
        tile_of[nat[nat >= 0]] = (np.arange(i.N_pad) // 128)[nat >= 0]
        ref_pairs = np.zeros((G, i.n_tiles), np.int64)
        for g in range(G):
            np.add.at(ref_pairs[g], tile_of, c_o.reshape(G, N)[g])
        np.testing.assert_array_equal(pairs.cpu().numpy(), ref_pairs)
        # block mask, lists ascending, full bits
        dense = gh.dense_block_mask(plan, mask)
        ref = oracle.block_mask(r_o, G, (T, H, W), gamma, Rt, (i.tile_h, i.tile_w), (i.tile_h, i.tile_w))
        np.testing.assert_array_equal(dense, ref)
        assert np.all(cnt.cpu().numpy() == (ref.reshape(G, i.n_tiles, -1) > 0).sum(-1))
        plan.close()


@pytest.mark.parametrize("c", CASES, ids=_ids)
@pytest.mark.parametrize("stride", [1, 3])
def test_entropy_matches_oracle(c, stride):
    T, H, W, G, d = c[:5]
    plan = _plan(c)
    i = plan.info
    if stride > i.n_tiles:
        pytest.skip("fewer tiles than the stride")
    q, k, _ = _qkv(c, 100 + sum(c[:5]))
    qt, kt = gh.to_tile_major(q, i), gh.to_tile_major(k, i)
    Ht = torch.empty(G, i.N_pad, device="cuda", dtype=torch.float32)
    plan.entropy(qt, kt, Ht, stride)
    torch.cuda.synchronize()
    assert plan.status() == 0
    Hn = gh.to_natural(Ht, i).cpu().numpy()
    ref = oracle.entropy(gh.bf16_bits(q), gh.bf16_bits(k), G, (T, H, W), d, key_stride=stride,
                         ktile=(i.tile_h, i.tile_w))
    gh.check_entropy(Hn.reshape(-1), ref)


def test_entropy_uniform_and_zero_query():
    # Q = 0 gives ln N exactly in the definition; the kernel must stay within tolerance
    c = (3, 17, 23, 2, 128, 0.8, 2, 8, 0)
    plan = _plan(c)
    i = plan.info
    k = torch.randn(2, i.N, 128, device="cuda").to(torch.bfloat16)
    q = torch.zeros_like(k)
    Ht = torch.empty(2, i.N_pad, device="cuda", dtype=torch.float32)
    for stride in (1, 2, 5):
        plan.entropy(gh.to_tile_major(q, i), gh.to_tile_major(k, i), Ht, stride)
        Hn = gh.to_natural(Ht, i).cpu().numpy()
        np.testing.assert_allclose(Hn, math.log(i.N), rtol=2e-5)


@pytest.mark.parametrize("c", CASES, ids=_ids)
def test_attention_matches_oracle(c):
    T, H, W, G, d, gamma, Rt, Bmin, _ = c
    N = T * H * W
    rng = np.random.default_rng(5 + sum(c[:5]))
    plan = _plan(c, 1.0, math.log(0.4))
    i = plan.info
    q, k, v = _qkv(c, 7 + sum(c[:5]))
    Hn = rng.uniform(0.0, math.log(N), size=(G, N)).astype(np.float32)
    mask = plan.new_mask()
    plan.radius_and_mask(gh.to_tile_major(torch.from_numpy(Hn).cuda(), i), mask)
    qt, kt, vt = (gh.to_tile_major(x, i) for x in (q, k, v))
    out = torch.full((G, i.N_pad, d), float("nan"), device="cuda", dtype=torch.float32)
    plan.attention(qt, kt, vt, mask, out)
    torch.cuda.synchronize()
    assert plan.status() == 0
    o = gh.to_natural(out, i).float().cpu().numpy().reshape(G * N, d)
    r_o, _, _ = oracle.radius(Hn.reshape(-1), G, (T, H, W), 1.0, math.log(0.4), gamma, Rt, Bmin)
    ref = oracle.attention(gh.bf16_bits(q), gh.bf16_bits(k), gh.bf16_bits(v), r_o, G, (T, H, W), d, gamma, Rt)
    gh.check_attention(o, ref)


@pytest.mark.parametrize("c", [CASES[0], CASES[2]], ids=_ids)
def test_attention_special_cases(c):
    """Self-only (Rt=0, tiny budget): O = V.  Dense (Rt=T-1, budget N): plain softmax attention."""
    T, H, W, G, d = c[:5]
    q, k, v = _qkv(c, 3)
    # self-only
    plan = tra.Plan(T, H, W, G, d, 1.0, -200.0, 0.8, 0, 1)
    i = plan.info
    mask = plan.new_mask()
    plan.radius_and_mask(torch.zeros(G, i.N_pad, device="cuda"), mask)
    out = plan.new_out()
    plan.attention(gh.to_tile_major(q, i), gh.to_tile_major(k, i), gh.to_tile_major(v, i), mask, out)
    o = gh.to_natural(out, i)
    assert torch.equal(o, v.float())
    # dense
    plan = tra.Plan(T, H, W, G, d, 1.0, 60.0, 0.8, T - 1, 1)
    i = plan.info
    mask = plan.new_mask()
    plan.radius_and_mask(torch.zeros(G, i.N_pad, device="cuda"), mask)
    _, cnt, pairs, _ = plan.mask_views(mask)
    assert int(pairs.sum()) == G * i.N * i.N
    assert torch.all(cnt == i.n_tiles)
    out = plan.new_out()
    plan.attention(gh.to_tile_major(q, i), gh.to_tile_major(k, i), gh.to_tile_major(v, i), mask, out)
    o = gh.to_natural(out, i).double()
    ref = torch.nn.functional.scaled_dot_product_attention(q.double()[None], k.double()[None], v.double()[None])[0]
    gh.check_attention(o.cpu().numpy(), ref.cpu().numpy())
    assert plan.status() == 0


@pytest.mark.parametrize("c", [CASES[0], CASES[2], CASES[6]], ids=_ids)
def test_pipeline_entropy_mask_attention(c):
    """The whole path on one set of inputs: GPU entropy -> GPU radius/mask (bit-exact
    given those entropies) -> GPU attention, against the oracle chain."""
    T, H, W, G, d, gamma, Rt, Bmin, _ = c
    N = T * H * W
    plan = _plan(c, 1.0, math.log(0.25))
    i = plan.info
    q, k, v = _qkv(c, 11)
    qt, kt, vt = (gh.to_tile_major(x, i) for x in (q, k, v))
    Ht = torch.empty(G, i.N_pad, device="cuda", dtype=torch.float32)
    mask = plan.new_mask()
    out = plan.new_out()
    plan.entropy(qt, kt, Ht)
    plan.radius_and_mask(Ht, mask)
    plan.attention(qt, kt, vt, mask, out)
    torch.cuda.synchronize()
    assert plan.status() == 0
    Hn = gh.to_natural(Ht, i).cpu().numpy().reshape(-1)
    qb, kb, vb = gh.bf16_bits(q), gh.bf16_bits(k), gh.bf16_bits(v)
    gh.check_entropy(Hn, oracle.entropy(qb, kb, G, (T, H, W), d))
    r_o, _, _ = oracle.radius(Hn, G, (T, H, W), 1.0, math.log(0.25), gamma, Rt, Bmin)
    rad = plan.mask_views(mask)[0].cpu().numpy()
    nat = gh.tile_major_index(i)
    r_gpu = np.zeros((G, N), np.int32)
    r_gpu[:, nat[nat >= 0]] = rad[:, nat >= 0]
    np.testing.assert_array_equal(r_gpu.reshape(-1), r_o)
    ref = oracle.attention(qb, kb, vb, r_o, G, (T, H, W), d, gamma, Rt)
    gh.check_attention(gh.to_natural(out, i).float().cpu().numpy().reshape(G * N, d), ref)


def test_mask_reuse_across_calls_with_fresh_v():
    """The mask is built once and reused ("Reutilisation Inter-Etapes"): later calls
    with new V must equal the oracle on that V."""
    c = CASES[2]
    T, H, W, G, d, gamma, Rt, Bmin, _ = c
    N = T * H * W
    plan = _plan(c, 1.0, math.log(0.3))
    i = plan.info
    q, k, _ = _qkv(c, 1)
    Hn = np.random.default_rng(0).uniform(0, math.log(N), size=(G, N)).astype(np.float32)
    mask = plan.new_mask()
    plan.radius_and_mask(gh.to_tile_major(torch.from_numpy(Hn).cuda(), i), mask)
    r_o, _, _ = oracle.radius(Hn.reshape(-1), G, (T, H, W), 1.0, math.log(0.3), gamma, Rt, Bmin)
    qt, kt = gh.to_tile_major(q, i), gh.to_tile_major(k, i)
    for call in range(3):
        v = synth.make_v(T, H, W, G, d, 1000 + call, device="cuda")
        out = plan.new_out()
        plan.attention(qt, kt, gh.to_tile_major(v, i), mask, out)
        ref = oracle.attention(gh.bf16_bits(q), gh.bf16_bits(k), gh.bf16_bits(v), r_o, G, (T, H, W), d, gamma, Rt)
        gh.check_attention(gh.to_natural(out, i).float().cpu().numpy().reshape(G * N, d), ref)


def test_argument_errors_on_device_calls():
    plan = _plan(CASES[0])
    i = plan.info
    x = plan.new_tile_major()
    o = plan.new_out()
    Ht = torch.empty(i.heads, i.N_pad, device="cuda")
    mask = plan.new_mask()
    with pytest.raises(tra.TraError) as e:
        tra.tra_radius_and_mask(plan.handle, Ht.data_ptr(), mask.data_ptr(), i.mask_bytes - 1)
    assert e.value.status == 3
    with pytest.raises(tra.TraError) as e:
        tra.tra_attention(plan.handle, x.data_ptr() + 2, x.data_ptr(), x.data_ptr(), mask.data_ptr(), o.data_ptr())
    assert e.value.status == 1
    with pytest.raises(tra.TraError) as e:
        tra.tra_entropy(plan.handle, x.data_ptr(), x.data_ptr(), Ht.data_ptr(), 0)
    assert e.value.status == 1
    with pytest.raises(tra.TraError) as e:
        tra.tra_attention(plan.handle, 0, x.data_ptr(), x.data_ptr(), mask.data_ptr(), o.data_ptr())
    assert e.value.status == 1
    with pytest.raises(tra.TraError) as e:
        tra.tra_permute(plan.handle, x.data_ptr(), o.data_ptr(), 1, 3)
    assert e.value.status == 1


def test_bounded_wait_gives_up_and_context_survives():
    """With the test hook every pipeline wait gives up at once: the kernels must
    record a timeout, drain their copies, free tensor memory and return; the
    next normal call must work and report OK."""
    c = CASES[2]
    T, H, W, G, d = c[:5]
    q, k, v = _qkv(c, 2)
    bad = _plan(c, flags=tra.TRA_FLAG_DEBUG_NO_WAIT)
    good = _plan(c)
    i = bad.info
    qt, kt, vt = (gh.to_tile_major(x, i) for x in (q, k, v))
    Ht = torch.empty(G, i.N_pad, device="cuda")
    mask = good.new_mask()
    good.entropy(qt, kt, Ht)
    good.radius_and_mask(Ht, mask)
    torch.cuda.synchronize()
    assert good.status() == 0
    out = good.new_out()
    bad.attention(qt, kt, vt, mask, out)
    torch.cuda.synchronize()
    assert bad.status() == 5
    bad.entropy(qt, kt, Ht)
    torch.cuda.synchronize()
    assert bad.status() == 5
    assert good.status() == 0            # the word was cleared by the read
    good.entropy(qt, kt, Ht)
    good.attention(qt, kt, vt, mask, out)
    torch.cuda.synchronize()
    assert good.status() == 0
    assert torch.isfinite(gh.to_natural(out, i).float()).all()


@pytest.mark.parametrize("extra", [tra.TRA_FLAG_QSORT, tra.TRA_FLAG_NATURAL, tra.TRA_FLAG_QSORT | tra.TRA_FLAG_DISK],
                         ids=["groups", "natural", "groups-disk"])
def test_bounded_wait_other_paths(extra):
    """The same give-up hook on the other code paths: radius-sorted groups (Q
    gathered before the roles start, no Q barrier), the natural layout (4-D
    TMA boxes), the disk, and the calibration kernel.  Each records a timeout
    and returns; a normal call afterwards works and reports OK."""
    T, H, W, G, d = 5, 17, 23, 2, 128
    flags = extra | tra.tra_flag_tile_w(8)
    good = tra.Plan(T, H, W, G, d, 1.0, math.log(0.3), 0.8, 3, 8, flags)
    bad = tra.Plan(T, H, W, G, d, 1.0, math.log(0.3), 0.8, 3, 8, flags | tra.TRA_FLAG_DEBUG_NO_WAIT)
    i = good.info
    q, k, v = synth.make_qkv(T, H, W, G, d, 13, device="cuda", dtype=torch.bfloat16)
    natural = bool(extra & tra.TRA_FLAG_NATURAL)
    qi, ki, vi = (q, k, v) if natural else (gh.to_tile_major(x, i) for x in (q, k, v))
    Ht = good.new_entropy() if natural else torch.empty(G, i.N_pad, device="cuda")
    mask, out = good.new_mask(), good.new_out()
    good.entropy(qi, ki, Ht)
    good.radius_and_mask(Ht, mask)
    torch.cuda.synchronize()
    assert good.status() == 0
    bad.attention(qi, ki, vi, mask, out)
    torch.cuda.synchronize()
    assert bad.status() == 5
    bad.calibrate_topk(qi, ki, 0.9, 2)
    torch.cuda.synchronize()
    assert bad.status() == 5
    good.attention(qi, ki, vi, mask, out)
    Hc, Kc = good.calibrate_topk(qi, ki, 0.9, 2)
    torch.cuda.synchronize()
    assert good.status() == 0
    o = out if natural else gh.to_natural(out, i)
    assert torch.isfinite(o.float()).all()
    assert int(Kc.max()) >= 1
    good.close()
    bad.close()


@pytest.mark.parametrize("c", [CASES[1], CASES[4]], ids=_ids)
def test_attention_bf16_output(c):
    """bf16 output: the fp32 result rounded once more; allowed error adds half a
    bf16 ulp of the reference value (2^-9 relative) to the fp32 bound."""
    T, H, W, G, d, gamma, Rt, Bmin, _ = c
    N = T * H * W
    plan = _plan(c, 1.0, math.log(0.4), flags=tra.TRA_FLAG_OUT_BF16)
    i = plan.info
    q, k, v = _qkv(c, 77)
    Hn = np.random.default_rng(4).uniform(0.0, math.log(N), size=(G, N)).astype(np.float32)
    mask = plan.new_mask()
    plan.radius_and_mask(gh.to_tile_major(torch.from_numpy(Hn).cuda(), i), mask)
    out = plan.new_out()
    assert out.dtype == torch.bfloat16
    plan.attention(*(gh.to_tile_major(x, i) for x in (q, k, v)), mask, out)
    torch.cuda.synchronize()
    o = gh.to_natural(out, i).double().cpu().numpy().reshape(G * N, d)
    r_o, _, _ = oracle.radius(Hn.reshape(-1), G, (T, H, W), 1.0, math.log(0.4), gamma, Rt, Bmin)
    ref = oracle.attention(gh.bf16_bits(q), gh.bf16_bits(k), gh.bf16_bits(v), r_o, G, (T, H, W), d, gamma, Rt)
    err = np.abs(o - ref)
    assert np.all(err <= gh.ATT_MAX + np.abs(ref) * 2.0 ** -9)
    assert err.mean() <= gh.ATT_MEAN + 2.0 ** -9 * np.abs(ref).mean()
