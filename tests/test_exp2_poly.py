"""The FMA-pipe exp2 used for part of the softmax exponentials: its constants and error bound.

The kernel's polynomial (exp2_poly in arl2_device.cuh) is checked here against the
mathematical 2^x. The check evaluates it step for step in float32 (round-to-nearest
split, single-rounding FMAs, exponent add) over the range the softmax uses.
"""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "softmax_attention_ar_b200", "csrc")


def _fit():
    spec = importlib.util.spec_from_file_location("fit_exp2_poly", os.path.join(CSRC, "fit_exp2_poly.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _kernel_coefficients():
    src = open(os.path.join(CSRC, "arl2_device.cuh")).read()
    body = src[src.index("float exp2_poly(float x)"):]
    body = body[: body.index("}")]
    nums = [float(v) for v in re.findall(r"(-?\d+\.\d+)f", body)]
    # fmaf(fmaf(fmaf(c3, f, c2), f, c1), f, c0) after the two 12582912 constants and -127
    c3, c2, c1, c0 = [v for v in nums if abs(v) < 2][-4:]
    return np.array([c0, c1, c2, c3], dtype=np.float32)


def test_kernel_constants_are_the_fitted_ones():
    fit = _fit()
    c = fit.remez(3).astype(np.float32)
    np.testing.assert_allclose(_kernel_coefficients(), c, rtol=2e-7)


def test_relative_error_bound():
    fit = _fit()
    c = _kernel_coefficients()
    xs = np.concatenate([np.linspace(-125, 64, 400_001, dtype=np.float32),
                         np.float32([0, -0.5, 0.5, -1, 1, 8, -8, -125, 64])])
    got = fit.eval_f32(c, xs).astype(np.float64)
    rel = np.abs(got / np.exp2(xs.astype(np.float64)) - 1)
    assert rel.max() < 1.5e-4
    low = fit.eval_f32(c, np.float32([-np.inf, -200.0, -126.0]))
    assert np.all(low >= 0) and np.all(low < 2.0 ** -125)   # masked scores vanish
