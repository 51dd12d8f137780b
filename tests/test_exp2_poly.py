"""The software 2^x of the attention softmax: the constants compiled into the kernels
are the ones the fitting script derives, and the algorithm (run in float32 by numpy
with the kernel's operation order) stays within 2e-4 relative of 2^x (CPU only)."""
import os
import re
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "block_sparse_long_prefill_b200", "csrc")
sys.path.insert(0, CSRC)
import exp2_poly  # noqa: E402


def test_constants_in_kernel_match_the_fit():
    text = open(os.path.join(CSRC, "common.cuh")).read()
    got = {int(k): float(v) for k, v in re.findall(r"kExp2C(\d) = ([0-9.e+-]+)f;", text)}
    coef = exp2_poly.coefficients()
    assert sorted(got) == [1, 2, 3]
    for j in (1, 2, 3):
        assert np.float32(got[j]) == np.float32(coef[j])


def test_relative_error_bound():
    coef = exp2_poly.coefficients()
    xs = np.concatenate([np.linspace(-126, 8, 2_000_001, dtype=np.float32),
                         np.arange(-20, 9, dtype=np.float32)])   # integers: f = 0 exactly
    got = exp2_poly.evaluate_f32(xs, coef).astype(np.float64)
    rel = np.abs(got / np.exp2(xs.astype(np.float64)) - 1)
    assert rel.max() < 2e-4
    # 2^n exactly at integers (p(0) = 1).
    ints = np.arange(-20, 9, dtype=np.float32)
    assert np.array_equal(exp2_poly.evaluate_f32(ints, coef), np.exp2(ints))


def test_masked_inputs_vanish():
    coef = exp2_poly.coefficients()
    out = exp2_poly.evaluate_f32(np.array([-np.inf, -1e30, -200.0], dtype=np.float32), coef)
    assert np.all(out < 1e-37) and np.all(out >= 0)
