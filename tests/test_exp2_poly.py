"""The FMA-pipe exp2 used for part of the softmax exponentials: range
reduction by the 1.5*2^23 (+127) rounding constant, a fitted polynomial on
[-1/2, 1/2], and a 2^k scale built from the same bits.  This emulates the
kernel's exact fp32 operation sequence in numpy (coefficients read from the
header) and checks the stated error bounds against exact 2^x, plus the edge
behaviour the kernels rely on (x <= -127 gives exactly 0)."""
import os
import re

import numpy as np
import pytest

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "sparse_attention_video_tra_b200", "csrc", "sm100.cuh")


def coeffs(deg):
    src = open(HDR).read()
    body = src[src.index("__device__ __forceinline__ float ex2_poly"):]
    branch = body[body.index("DEG == 3"):body.index("} else {")] if deg == 3 else \
        body[body.index("} else {"):body.index("const float scale")]
    vals = [np.float32(v) for v in re.findall(r"(\d+\.\d+)f", branch)]
    # Horner nesting lists the highest coefficient first
    return vals


def fma32(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def ex2_poly(x, deg):
    x = np.maximum(np.asarray(x, np.float32), np.float32(-127.0))
    C = np.float32(12583039.0)
    t = (x + C).astype(np.float32)
    f = (x - (t - C).astype(np.float32)).astype(np.float32)
    cs = coeffs(deg)
    p = np.full_like(f, cs[0])
    for c in cs[1:]:
        p = fma32(p, f, np.full_like(f, c))
    bits = (t.view(np.int32).astype(np.int64) << 23).astype(np.uint64) & np.uint64(0xFFFFFFFF)
    scale = bits.astype(np.uint32).view(np.float32)
    return (p * scale).astype(np.float32)


@pytest.mark.parametrize("deg,bound", [(3, 7.6e-5), (4, 2.8e-6)])
def test_relative_error_bound(deg, bound):
    x = np.concatenate([np.linspace(-120, 8, 2_000_001), np.linspace(-1, 1, 200_001)]).astype(np.float32)
    y = ex2_poly(x, deg).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1)
    assert rel.max() <= bound, rel.max()


@pytest.mark.parametrize("deg", [3, 4])
def test_underflow_and_masked_inputs_give_zero(deg):
    x = np.array([-np.inf, -1e30, -1000.0, -127.0, -130.5], np.float32)
    assert np.all(ex2_poly(x, deg) == 0.0)
    # just above the cut the result is a normal number close to 2^x
    y = ex2_poly(np.array([-126.0, -100.25, 0.0, 7.5], np.float32), deg)
    np.testing.assert_allclose(y, np.exp2([-126.0, -100.25, 0.0, 7.5]), rtol=1e-4)


def test_coefficients_parse():
    assert len(coeffs(3)) == 4 and len(coeffs(4)) == 5
    assert abs(coeffs(3)[-1] - 1) < 1e-3 and abs(coeffs(4)[-2] - np.log(2)) < 1e-3


def pair_coeffs():
    src = open(HDR).read()
    body = src[src.index("ex2_poly4_pair"):]
    body = body[:body.index("return f2_mul")]
    vals = re.findall(r"f2_pack\((\d+\.\d+)f, \1f\)", body)
    return [np.float32(v) for v in vals if float(v) < 1.5 and v not in ("1.0",)]


def ex2_pair(x):
    """The packed-pair variant: f = x + (C - t) instead of x - (t - C)."""
    x = np.maximum(np.asarray(x, np.float32), np.float32(-127.0))
    C = np.float32(12583039.0)
    t = (x + C).astype(np.float32)
    f = (x + fma32(t, np.full_like(t, np.float32(-1.0)), np.full_like(t, C))).astype(np.float32)
    cs = pair_coeffs()
    p = fma32(np.full_like(f, cs[0]), f, np.full_like(f, cs[1]))
    for c in cs[2:]:
        p = fma32(p, f, np.full_like(f, c))
    bits = (t.view(np.int32).astype(np.int64) << 23).astype(np.uint64) & np.uint64(0xFFFFFFFF)
    return (p * bits.astype(np.uint32).view(np.float32)).astype(np.float32)


def test_pair_variant_matches_scalar_coefficients_and_bound():
    assert [float(c) for c in pair_coeffs()] == [float(c) for c in coeffs(4)]
    x = np.linspace(-120, 0, 1_000_001).astype(np.float32)
    rel = np.abs(ex2_pair(x).astype(np.float64) / np.exp2(x.astype(np.float64)) - 1)
    assert rel.max() <= 2.8e-6
    assert np.all(ex2_pair(np.array([-np.inf, -1e30, -127.0], np.float32)) == 0.0)
