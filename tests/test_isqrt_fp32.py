"""The disk half-width isqrt(s^2 - dh^2) is taken on the GPU as the floor of a
correctly rounded fp32 square root.  For every integer n in [0, 1023^2] (the
range the kernels reach: half-widths are clamped at 1023) that floor equals
the exact integer square root; numpy's float32 sqrt is correctly rounded as
CUDA's sqrtf is without fast-math."""
import math

import numpy as np


def test_floor_of_fp32_sqrt_is_exact_isqrt_up_to_1023_squared():
    n = np.arange(0, 1023 * 1023 + 1, dtype=np.int64)
    got = np.floor(np.sqrt(n.astype(np.float32))).astype(np.int64)
    k = np.array([math.isqrt(int(v)) for v in range(0, 1023 * 1023 + 1, 997)], dtype=np.int64)
    np.testing.assert_array_equal(got[::997], k)
    # the exact property for all n: k^2 <= n < (k+1)^2
    assert np.all(got * got <= n) and np.all((got + 1) * (got + 1) > n)
