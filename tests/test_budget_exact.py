"""The budget's ceiling is exact: Bhat = ceil(min(N, max(Bmin, e^y))) with
y = a*H + b ("Token Radius Attention for Efficient Video Generation",
gist.science summary, section 2, Intuition I: B ~ tau*exp(H_i)).

For a double y != 0, e^y is irrational, so its ceiling has one answer even
when e^y lies within an ulp of an integer -- which it does for a whole class
of plans: a = 0, b = ln k (a fixed budget of k tokens).  The oracle evaluates
e^y in binary128; it is pinned here against Python's decimal arithmetic at 60
digits.  The library's rule (an fp64 exponential, re-decided in double-double
arithmetic within 16 ulps of an integer) is built for the host from the same
source the kernel uses and compared with the oracle on the same exponents."""
import math
import os
import subprocess
from decimal import Decimal, getcontext

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "sparse_attention_video_tra_b200", "csrc")
BIG_N = 1 << 31


def exact_ceil_exp(y: float) -> int:
    getcontext().prec = 60
    return int(Decimal(y).exp().to_integral_value(rounding="ROUND_CEILING"))


def near_integer_exponents():
    """fp64(ln k) and its neighbours up to 3 ulps either side, k = 2..2500,
    plus the same around k = 10^4 .. 10^9."""
    ys = []
    ks = list(range(2, 2501)) + [10 ** p + d for p in range(4, 10) for d in (-1, 0, 1)]
    for k in ks:
        y = math.log(k)
        for step in range(-3, 4):
            v = y
            for _ in range(abs(step)):
                v = math.nextafter(v, math.inf if step > 0 else -math.inf)
            ys.append(v)
    return ys


def test_oracle_budget_is_the_exact_ceiling_near_integers():
    ys = near_integer_exponents()
    bad = [(y, oracle.budget(0.0, 0.0, y, BIG_N, 1), exact_ceil_exp(y)) for y in ys
           if oracle.budget(0.0, 0.0, y, BIG_N, 1) != exact_ceil_exp(y)]
    assert not bad, bad[:5]
    # the band matters: a plain fp64 exponential misses some of these
    assert sum(math.ceil(math.exp(y)) != exact_ceil_exp(y) for y in ys) > 0


def test_oracle_budget_clamps_and_special_cases():
    assert oracle.budget(0.0, 0.0, 0.0, 1000, 1) == 1                 # e^0 = 1 exactly
    assert oracle.budget(0.0, 0.0, 1e-300, 1000, 1) == 2              # just above 1
    assert oracle.budget(0.0, 0.0, -5.0, 1000, 7) == 7                # below Bmin
    assert oracle.budget(0.0, 0.0, 50.0, 1000, 7) == 1000             # above N
    assert oracle.budget(0.0, 0.0, float("nan"), 1000, 7) == 7
    assert oracle.budget(0.0, 0.0, math.log(1000.5), 1000, 1) == 1000


@pytest.fixture(scope="module")
def harness(tmp_path_factory):
    exe = str(tmp_path_factory.mktemp("budget") / "exact_budget_harness")
    subprocess.run(["g++", "-O2", "-std=c++17", "-ffp-contract=off", "-I", CSRC, "-I", "/usr/local/cuda/include",
                    os.path.join(ROOT, "tests", "exact_budget_harness.cpp"), "-o", exe, "-lm"], check=True)
    return exe


def _library_budgets(exe, ys, N, Bmin):
    inp = "".join(f"{float(y).hex()} {N} {Bmin}\n" for y in ys)
    out = subprocess.run([exe], input=inp, capture_output=True, text=True, check=True).stdout.split()
    return [int(x) for x in out]


def test_library_rule_equals_oracle_near_integers(harness):
    ys = near_integer_exponents()
    got = _library_budgets(harness, ys, BIG_N, 1)
    ref = [oracle.budget(0.0, 0.0, y, BIG_N, 1) for y in ys]
    assert got == ref


def test_library_rule_equals_oracle_on_random_exponents(harness):
    rng = np.random.default_rng(5)
    ys = list(rng.uniform(-3.0, 23.0, 20000)) + [0.0, -0.0, 1e-300, -1e-300, 700.0, -700.0, float("nan")]
    for N, Bmin in ((BIG_N, 1), (75600, 8), (256, 8)):
        got = _library_budgets(harness, ys, N, Bmin)
        ref = [oracle.budget(0.0, 0.0, y, N, Bmin) for y in ys]
        assert got == ref
