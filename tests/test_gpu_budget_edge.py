"""GPU radii where the budget's exponential sits on an integer.

With y = a*H + b swept across fp64(ln k) a few ulps at a time (a = 2^-52, H
in [0, 64], b eight ulps below ln k), e^y crosses the integer k inside the
sweep, so Bhat is k for some queries and k + 1 for others; an exponential
one ulp off on either side would put some of them on the wrong side.  On a
one-frame grid an interior query's count is (2r + 1)^2, so for k = (2r+1)^2
the two budgets give different radii.  The kernel's radii must equal the
oracle's (exact ceiling, binary128) bit for bit.  "Token Radius Attention
for Efficient Video Generation" (gist.science summary), section 2,
Intuition I (B ~ tau*exp(H)) and "Budget-vers-Rayon"."""
import math

import numpy as np
import pytest
import torch

import oracle
import sparse_attention_video_tra_b200 as tra
from sparse_attention_video_tra_b200 import build as trabuild
import gpu_helpers as gh

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    trabuild.build()
    yield


@pytest.mark.parametrize("k", [9, 25, 49, 81, 121, 169, 225, 289, 26, 50, 100, 1000])
def test_radii_bit_exact_when_the_budget_is_on_an_integer(k):
    T, H, W, G, d = 1, 40, 40, 2, 64
    N = T * H * W
    a = 2.0 ** -52
    y0 = math.log(k)
    ulp = math.ulp(y0)
    b = y0 - 8 * ulp
    plan = tra.Plan(T, H, W, G, d, a, b, 0.8, 0, 1)
    i = plan.info
    rng = np.random.default_rng(k)
    Hn = rng.uniform(0.0, 64.0 * ulp / (2.0 ** -52) / 4.0, size=(G, N)).astype(np.float32)
    Hn = np.minimum(Hn, np.float32(64.0))
    Ht = gh.to_tile_major(torch.from_numpy(Hn).cuda(), i)
    mask = plan.new_mask()
    plan.radius_and_mask(Ht, mask)
    torch.cuda.synchronize()
    assert plan.status() == 0
    nat = gh.tile_major_index(i)
    rad = plan.mask_views(mask)[0].cpu().numpy()
    r_gpu = np.zeros((G, N), np.int32)
    r_gpu[:, nat[nat >= 0]] = rad[:, nat >= 0]
    r_o, _, bh = oracle.radius(Hn.reshape(-1), G, (T, H, W), a, b, 0.8, 0, 1)
    # the sweep straddles the integer: both budgets occur
    assert set(np.unique(bh)) == {k, k + 1}, np.unique(bh)
    np.testing.assert_array_equal(r_gpu.reshape(-1), r_o)
    plan.close()
