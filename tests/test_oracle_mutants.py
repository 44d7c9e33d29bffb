"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of oracle/tra_oracle.c (a dropped
term, an off-by-one bound, a strict comparison, a wrong log base or sign),
compiles it, and runs the pin tests that should notice with that library
loaded instead of the real one: they must fail.  A control run of the same
harness on the unchanged source must pass.  Only the copy is changed; the
oracle itself is never modified."""
import os
import subprocess
import sys

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PINS = "tests/test_oracle_pins.py"
DISK = "tests/test_oracle_disk_pins.py"
CALIB = "tests/test_oracle_calibration_pins.py"

# (what is wrong, text in tra_oracle.c, replacement, which occurrence, pin tests)
MUTANTS = [
    ("half-width loses the 1e-9", "volatile double sum = prod + EPS_S;", "volatile double sum = prod;", 1,
     [f"{PINS}::test_halfwidth_closed_forms", f"{PINS}::test_count_golden"]),
    ("r_cap one short", "while (oracle_halfwidth(r, g) < need) ++r;", "while (oracle_halfwidth(r, g) < need - 1) ++r;",
     1, [f"{PINS}::test_rt_eff_and_r_cap"]),
    ("temporal reach one frame short", "for (int dt = -rte; dt <= rte; ++dt) {", "for (int dt = -rte; dt < rte; ++dt) {",
     1, [f"{PINS}::test_count_equals_bruteforce_mask_rows"]),
    ("budget floored instead of ceiled", "__float128 c = ceilq(expq((__float128)x));",
     "__float128 c = floorq(expq((__float128)x));", 1,
     [f"{PINS}::test_budget_closed_forms"]),
    ("radius scan stops one early", "while (c < bh && r < rcap) {", "while (c < bh - 1 && r < rcap) {", 1,
     [f"{PINS}::test_radius_matches_bruteforce"]),
    ("Chebyshev test strict", "return cheb <= s;", "return cheb < s;", 1,
     [f"{PINS}::test_block_mask_matches_bruteforce", f"{PINS}::test_attention_matches_bruteforce"]),
    ("disk test strict", "return dh * dh + dw * dw <= s * s;", "return dh * dh + dw * dw < s * s;", 1,
     [f"{DISK}::test_block_mask_matches_bruteforce", f"{DISK}::test_attention_matches_bruteforce"]),
    ("disk row width off by one", "c += imin64(W - 1, w + half) - imax64(0, w - half) + 1;",
     "c += imin64(W - 1, w + half) - imax64(0, w - half);", 1, [f"{DISK}::test_interior_count_is_gauss_circle_number"]),
    ("block mask never marks full", "(uint8_t)(any ? (all ? 3 : 1) : 0)", "(uint8_t)(any ? 1 : 0)", 1,
     [f"{PINS}::test_block_mask_matches_bruteforce"]),
    ("entropy in bits", "H_out[row] = log(Z) - S / Z + corr;", "H_out[row] = log2(Z) - S / Z + corr;", 1,
     [f"{PINS}::test_entropy_two_point_closed_form"]),
    ("subsample correction inverted", "log((double)N / (double)nS)", "log((double)nS / (double)N)", 1,
     [f"{PINS}::test_entropy_q_zero_subsampled_keeps_log_n"]),
    ("attention without the 1/sqrt(d) scale", "double sigma = 1.0 / sqrt((double)d);", "double sigma = 1.0;", 2,
     [f"{PINS}::test_dense_case_equals_sdpa"]),
    ("set block mask never marks full", "out[set * nK + kb] = (uint8_t)(some && any ? (all ? 3 : 1) : 0);",
     "out[set * nK + kb] = (uint8_t)(some && any ? 1 : 0);", 1,
     ["tests/test_oracle_qsort_pins.py::test_sets_equal_tiles_when_sets_are_tiles",
      "tests/test_oracle_qsort_pins.py::test_sets_equal_bruteforce"]),
    ("calibration cut one key late", "if (cum >= mass) { kk = j + 1; break; }", "if (cum > mass) { kk = j + 2; break; }", 1,
     [f"{CALIB}::test_uniform_attention_needs_ceil_mass_times_n", f"{CALIB}::test_topk_matches_numpy_sort"]),
    ("budget ceiling from an fp64 exponential", "__float128 c = ceilq(expq((__float128)x));",
     "__float128 c = ceilq((__float128)exp(x));", 1,
     ["tests/test_budget_exact.py::test_oracle_budget_is_the_exact_ceiling_near_integers"]),
    ("calibration fit through the origin (no intercept)", "double dx = H[i] - mx, dy = fit_y(k[i]) - my;",
     "double dx = H[i], dy = fit_y(k[i]);", 1,
     [f"{CALIB}::test_fit_hand_worked_three_points", f"{CALIB}::test_fit_matches_numpy_polyfit_on_noisy_data"]),
    ("calibration fit in log2", "static double fit_y(int64_t k) { return log((double)k); }",
     "static double fit_y(int64_t k) { return log2((double)k); }", 1,
     [f"{CALIB}::test_fit_hand_worked_three_points", f"{CALIB}::test_fit_recovers_exact_log_linear_data"]),
    ("calibration fit regresses H on ln k", "*a_out = sxy / sxx;", "*a_out = syy / sxy;", 1,
     [f"{CALIB}::test_fit_hand_worked_three_points", f"{CALIB}::test_fit_matches_numpy_polyfit_on_noisy_data"]),
]


def _replace_nth(text, old, new, n):
    at = -1
    for _ in range(n):
        at = text.index(old, at + 1)
    return text[:at] + new + text[at + len(old):]


def _run_pins(lib, tests):
    env = dict(os.environ, TRA_ORACLE_LIB=str(lib))
    return subprocess.run([sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider", "-m", "not gpu", *tests],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)


def test_control_unchanged_source_passes(tmp_path):
    src = open(oracle._SRC).read()
    path = tmp_path / "same.c"
    path.write_text(src)
    lib = oracle.compile_source(str(path), str(tmp_path / "libsame.so"))
    tests = sorted({t for m in MUTANTS for t in m[4]})
    p = _run_pins(lib, tests)
    assert p.returncode == 0, p.stdout[-2000:]


@pytest.mark.parametrize("what,old,new,nth,tests", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_reject_planted_mistake(tmp_path, what, old, new, nth, tests):
    src = open(oracle._SRC).read()
    assert src.count(old) >= nth, f"mutation site not found: {old}"
    path = tmp_path / "mutant.c"
    path.write_text(_replace_nth(src, old, new, nth))
    lib = oracle.compile_source(str(path), str(tmp_path / "libmutant.so"))
    p = _run_pins(lib, tests)
    assert p.returncode == 1, f"the pins did not catch: {what}\n{p.stdout[-2000:]}"
