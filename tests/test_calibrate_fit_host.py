"""The library's calibration fit (tra_calibrate_fit: host code behind the C
ABI) against the oracle's fit on the same (H, k) rows.  "Token Radius
Attention for Efficient Video Generation" (gist.science summary), section 2,
Intuition I: ln k = a*H + b, the tau*exp(H) law with a free slope.  No GPU."""
import math

import numpy as np
import pytest

import oracle
import sparse_attention_video_tra_b200 as tra
from sparse_attention_video_tra_b200 import build as trabuild
from sparse_attention_video_tra_b200.calibrate import fit_log_linear


@pytest.fixture(scope="module", autouse=True)
def built():
    trabuild.build()
    yield


def _pairs(seed, n, a=1.1, b=-0.3, noise=0.5):
    rng = np.random.default_rng(seed)
    H = rng.uniform(1.0, 11.0, n).astype(np.float32)
    k = np.maximum(1, np.round(np.exp(a * H.astype(np.float64) + b + rng.normal(0, noise, n)))).astype(np.int32)
    return H, k


@pytest.mark.parametrize("seed,n", [(1, 2), (2, 3), (3, 100), (4, 5000), (5, 200000)])
def test_library_fit_equals_oracle_fit(seed, n):
    H, k = _pairs(seed, n)
    a, b = fit_log_linear(H, k)
    ao, bo, _, m = oracle.fit_log_linear(H.astype(np.float64), k)
    assert m == n
    assert a == pytest.approx(ao, rel=1e-9, abs=1e-12)
    assert b == pytest.approx(bo, rel=1e-9, abs=1e-11)


def test_library_fit_hand_worked_case_and_pad_rows():
    # x = (0, 1, 2), k = (1, 2, 8): a = (3/2) ln 2, b = -(1/6) ln 2 (derived by
    # hand in the oracle's pins); pad rows of tra_calibrate_topk (NaN, -1) drop out
    H = np.array([0.0, np.nan, 1.0, 2.0, 7.0], np.float32)
    k = np.array([1, -1, 2, 8, -1], np.int32)
    a, b, m = tra.tra_calibrate_fit(H.ctypes.data, k.ctypes.data, H.size)
    assert m == 3
    assert a == pytest.approx(1.5 * math.log(2.0), rel=1e-14)
    assert b == pytest.approx(-math.log(2.0) / 6.0, rel=1e-12)


def test_library_fit_rejects_degenerate_input():
    for H, k in (([1.0], [3]), ([2.0, 2.0, 2.0], [1, 4, 9]), ([1.0, 2.0], [0, 5])):
        with pytest.raises(tra.TraError) as e:
            fit_log_linear(np.array(H, np.float32), np.array(k, np.int32))
        assert e.value.status == 1
    with pytest.raises(tra.TraError):
        tra.tra_calibrate_fit(None, None, 3)
