"""The polynomial 2^x used for part of the prefill softmax (CPU checks).

The kernel computes some exponentials as 2^floor(x) * p(frac(x)) with a cubic
p fitted in exact_io_aware_101_b200/exp2_poly.py.  These tests re-run the fit,
check that the constants compiled into common.cuh are the fitted ones, and
bound the relative error of a float32 model of the whole evaluation against
numpy's exp2 over the range the softmax uses.
"""
import os
import re

import numpy as np

from exact_io_aware_101_b200 import exp2_poly

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def compiled_constants():
    src = open(os.path.join(ROOT, "exact_io_aware_101_b200", "csrc", "common.cuh")).read()
    out = []
    for name in ("kC0", "kC1", "kC2", "kC3"):
        m = re.search(name + r"\s*=\s*([0-9a-fx.p+-]+)f", src)
        assert m, name
        out.append(np.float32(float.fromhex(m.group(1))))
    return np.array(out, dtype=np.float32)


def test_constants_match_the_fit():
    np.testing.assert_array_equal(compiled_constants(), exp2_poly.fit())


def test_cubic_relative_error_on_unit_interval():
    f = np.linspace(0, 1, 100001, dtype=np.float32)[:-1]
    p = exp2_poly.horner_f32(compiled_constants(), f).astype(np.float64)
    rel = np.abs(p - np.exp2(f.astype(np.float64))) / np.exp2(f.astype(np.float64))
    assert rel.max() < 2.0 ** -13


def test_full_exp2_model_error_bound():
    x = np.concatenate([np.linspace(-126, 8, 1000001), [-0.0, 0.0, 1.0, -1.0, 7.999, -125.5]])
    x = x.astype(np.float32)
    y = exp2_poly.exp2_model(x, compiled_constants()).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() < 2.0 ** -12  # far inside bf16's 2^-8 relative step
    # Below the clamp the value is negligible, never negative or NaN.
    lo = exp2_poly.exp2_model(np.array([-200.0, -1e30, -np.inf], np.float32), compiled_constants())
    assert np.all(lo >= 0) and np.all(lo < 2.0 ** -124) and np.all(np.isfinite(lo))
