"""GPU calibration workload (tra_calibrate_topk) against the oracle.

"Token Radius Attention for Efficient Video Generation" (gist.science
summary), section 2, Intuition I: the key density a query needs follows its
entropy.  The kernel returns, for the queries of every s-th tile, the dense
entropy (bit for bit the entropy kernel's) and k_i, the fewest top keys
holding `mass` of the query's attention, by bisection on a score threshold.

k_i is an integer decided by floating point: the kernel's fp32 scores can
order near-equal probabilities differently from the oracle's exact ones, so
k_i is checked for validity against the oracle's sorted fp64 probabilities
(the top k_i keys hold at least mass - eps, the top k_i - 1 less than
mass + eps) and must equal the oracle's count on all but a small share of
rows; the log-linear fit from GPU pairs matches the fit from oracle pairs."""
import math

import numpy as np
import pytest
import torch

import oracle
import sparse_attention_video_tra_b200 as tra
from sparse_attention_video_tra_b200 import build as trabuild
from sparse_attention_video_tra_b200 import synth
from sparse_attention_video_tra_b200.calibrate import fit_log_linear
import gpu_helpers as gh

pytestmark = pytest.mark.gpu

CASES = [
    (4, 8, 8, 2, 64, 0.7, 2, 8, 0),
    (3, 17, 23, 2, 128, 0.8, 3, 8, 0),
    (3, 30, 52, 1, 128, 0.8, 2, 8, 4),
]
EPS = 1e-4


@pytest.fixture(scope="module", autouse=True)
def built():
    trabuild.build()
    yield


def _ids(c):
    return "x".join(map(str, c[:3])) + f"-d{c[4]}-tw{c[8]}"


def _plan(c, flags=0):
    T, H, W, G, d, gamma, Rt, Bmin, tw = c
    return tra.Plan(T, H, W, G, d, 1.0, 0.0, gamma, Rt, Bmin, flags | (tra.tra_flag_tile_w(tw) if tw else 0))


def _sorted_cum(q, k, d, g, n):
    s = (q[g, n].astype(np.float64) @ k[g].astype(np.float64).T) / math.sqrt(d)
    p = np.exp(s - s.max())
    p /= p.sum()
    return np.cumsum(-np.sort(-p))


@pytest.mark.parametrize("c", CASES, ids=_ids)
@pytest.mark.parametrize("mass,stride", [(0.9, 1), (0.5, 2)])
def test_calibration_counts_and_entropies(c, mass, stride):
    T, H, W, G, d = c[:5]
    N = T * H * W
    plan = _plan(c)
    i = plan.info
    q, k, _ = synth.make_qkv(T, H, W, G, d, 50 + sum(c[:5]), device="cuda", dtype=torch.bfloat16)
    qt, kt = gh.to_tile_major(q, i), gh.to_tile_major(k, i)
    Hc, Kc = plan.calibrate_topk(qt, kt, mass, stride)
    Ht = torch.empty(G, i.N_pad, device="cuda")
    plan.entropy(qt, kt, Ht, 1)
    torch.cuda.synchronize()
    assert plan.status() == 0
    n_sample = -(-i.n_tiles // stride)
    assert Hc.shape == (G, n_sample, 128)
    nat = gh.tile_major_index(i)
    rows = np.concatenate([np.arange(s * stride * 128, s * stride * 128 + 128) for s in range(n_sample)])
    Hc, Kc = Hc.cpu().numpy().reshape(G, -1), Kc.cpu().numpy().reshape(G, -1)
    He = Ht.cpu().numpy()[:, rows]
    valid = nat[rows] >= 0
    # entropies: the entropy kernel's, bit for bit; pad rows NaN / -1
    np.testing.assert_array_equal(Hc[:, valid], He[:, valid])
    assert np.all(np.isnan(Hc[:, ~valid])) and np.all(Kc[:, ~valid] == -1)
    # counts: valid against the exact sorted probabilities
    qb, kb = gh.bf16_bits(q), gh.bf16_bits(k)
    qf = q.float().cpu().numpy()
    kf = k.float().cpu().numpy()
    rng = np.random.default_rng(1)
    cols = np.nonzero(valid)[0]
    pick = cols if cols.size <= 200 else np.sort(rng.choice(cols, 200, replace=False))
    queries = np.array([g * N + nat[rows[j]] for g in range(G) for j in pick])
    ref = oracle.topk_count(qb, kb, G, (T, H, W), d, mass, queries=queries).reshape(G, -1)
    mismatch = 0
    for g in range(G):
        for t, j in enumerate(pick):
            kk = int(Kc[g, j])
            cum = _sorted_cum(qf, kf, d, g, nat[rows[j]])
            assert 1 <= kk <= N
            assert cum[kk - 1] >= mass - EPS
            assert kk == 1 or cum[kk - 2] < mass + EPS
            mismatch += kk != ref[g, t]
    assert mismatch <= max(1, 0.02 * ref.size)


def test_fit_matches_oracle_fit_and_natural_layout():
    c = (3, 17, 23, 2, 128, 0.8, 3, 8, 0)
    T, H, W, G, d = c[:5]
    N = T * H * W
    tm, nat = _plan(c), _plan(c, tra.TRA_FLAG_NATURAL)
    i = tm.info
    q, k, _ = synth.make_qkv(T, H, W, G, d, 91, device="cuda", dtype=torch.bfloat16)
    Ht, Kt = tm.calibrate_topk(gh.to_tile_major(q, i), gh.to_tile_major(k, i), 0.9, 1)
    Hn, Kn = nat.calibrate_topk(q, k, 0.9, 1)
    torch.cuda.synchronize()
    assert tm.status() == 0 and nat.status() == 0
    assert torch.equal(Kt, Kn) and torch.equal(torch.nan_to_num(Ht, 7.0), torch.nan_to_num(Hn, 7.0))
    a_g, b_g = fit_log_linear(Ht.cpu().numpy(), Kt.cpu().numpy())
    nat_idx = gh.tile_major_index(i)
    Hr = oracle.entropy(gh.bf16_bits(q), gh.bf16_bits(k), G, (T, H, W), d)
    Kr = oracle.topk_count(gh.bf16_bits(q), gh.bf16_bits(k), G, (T, H, W), d, 0.9)
    a_o, b_o, _, _ = oracle.fit_log_linear(Hr, Kr)           # the oracle's own fit on its own pairs
    assert abs(a_g - a_o) < 0.02 and abs(b_g - b_o) < 0.1
    assert a_g > 0.0                 # more entropy, more keys needed


def test_calibration_rejects_bad_arguments():
    plan = _plan(CASES[0])
    q = plan.new_tile_major()
    for mass, stride in ((0.0, 1), (1.0, 1), (0.9, 0)):
        with pytest.raises(tra.TraError) as e:
            plan.calibrate_topk(q, q, mass, stride) if stride else tra.tra_calibrate_topk(
                plan.handle, q.data_ptr(), q.data_ptr(), mass, stride, q.data_ptr(), q.data_ptr())
        assert e.value.status == 1
