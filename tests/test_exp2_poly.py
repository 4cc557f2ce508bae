"""The forward kernel's FMA-pipe exponential (sta_common.cuh, exp2_fma2),
checked on the CPU: its coefficients are the library's own minimax fit
(fit_exp2_poly.py reproduces them), and evaluated in float32 exactly as the
kernel evaluates it, it stays within the stated relative error of 2^x over
the range the softmax uses (x in [-126, 8]; inputs below are clamped)."""
import os
import re
import sys

import numpy as np

from sparse_local_attention_b200 import _build

sys.path.insert(0, _build.CSRC)
import fit_exp2_poly  # noqa: E402


def kernel_coefficients():
    src = open(os.path.join(_build.CSRC, "sta_common.cuh")).read()
    return np.array([float(re.search(rf"kExp2C{k} = ([0-9.eE+-]+)f;", src).group(1)) for k in range(4)],
                    dtype=np.float32)


def test_coefficients_are_the_minimax_fit():
    coef, level = fit_exp2_poly.remez()
    assert level < 8e-5
    np.testing.assert_array_equal(coef.astype(np.float32), kernel_coefficients())


def test_relative_error_against_exp2():
    c = kernel_coefficients()
    x = np.concatenate([np.linspace(-126.0, 8.0, 1_000_001, dtype=np.float32),
                        np.linspace(-0.5, 0.5, 100_001, dtype=np.float32),
                        np.arange(-126, 9, dtype=np.float32)])          # exact integers: r = 0
    got = fit_exp2_poly.kernel_exp2(x, c).astype(np.float64)
    rel = np.abs(got / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() <= 1.5e-4
    assert rel[x >= -125].max() <= 7.5e-5
    # far below the bf16 rounding of the probabilities (2^-9 relative)
    assert rel.max() < 2.0 ** -9 / 10


def test_clamp_and_rounding_edges():
    c = kernel_coefficients()
    # below the clamp: 2^-126 times p(0), positive and tiny (never negative or huge)
    low = fit_exp2_poly.kernel_exp2(np.array([-126.0, -127.0, -1e4, -np.inf], dtype=np.float32), c)
    assert np.all(low > 0) and np.all(low < 1.2e-38)
    # halfway points round to even: r stays within [-1/2, 1/2]
    half = np.array([-2.5, -1.5, -0.5, 0.5, 1.5, 7.5], dtype=np.float32)
    rel = np.abs(fit_exp2_poly.kernel_exp2(half, c) / np.exp2(half.astype(np.float64)) - 1.0)
    assert rel.max() <= 7.5e-5
