"""The polynomial 2^x used for part of the prefill softmax (CPU checks).

The kernel computes some exponentials as 2^floor(x) * p(frac(x)) with a cubic
p fitted in exact_io_aware_101_b200/exp2_poly.py.  These tests re-run the fit,
check that the constants compiled into common.cuh are the fitted ones, and
bound the relative error of a float32 model of the whole evaluation against
numpy's exp2 over the range the softmax uses; on the GPU, the device function
itself is evaluated (through the test build's probe) against CUDA's exp2f and
the float32 model.
"""
import os
import re

import numpy as np
import pytest

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


@pytest.mark.gpu
def test_device_exp2_poly_against_exp2f():
    # The device function itself (exp2_poly2, the packed two-wide form the
    # softmax calls), evaluated by the test build's probe over [-126, 0] -- the
    # range of s*c - m in the softmax -- against CUDA's exp2f on the same
    # inputs and against the float32 model above.
    import ctypes

    import torch

    import exact_io_aware_101_b200 as ea
    from exact_io_aware_101_b200 import build as eabuild

    lib = ea.load_library(eabuild.build_test_lib())
    lib.attn_test_exp2_poly.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int, ctypes.c_void_p]
    lib.attn_test_exp2_poly.restype = ctypes.c_int
    xs = np.concatenate([np.linspace(-126, 0, 2000001), [-0.0, -1.0, -125.5, -126.0],
                         -np.random.default_rng(0).random(1001) * 126]).astype(np.float32)
    x = torch.from_numpy(xs).cuda()
    y = torch.empty_like(x)
    ref = torch.empty_like(x)
    assert lib.attn_test_exp2_poly(x.data_ptr(), y.data_ptr(), ref.data_ptr(), x.numel(),
                                   torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    yd = y.cpu().numpy().astype(np.float64)
    rd = ref.cpu().numpy().astype(np.float64)
    exact = np.exp2(xs.astype(np.float64))
    assert np.all(np.isfinite(yd)) and np.all(yd > 0)
    assert (np.abs(yd - rd) / rd).max() < 2.0 ** -12
    assert (np.abs(yd - exact) / exact).max() < 2.0 ** -12
    # The device evaluation is the float32 model (whose fused multiply-adds are
    # emulated through float64, so a double rounding may differ by one unit in
    # the last place).
    model = exp2_poly.exp2_model(xs, compiled_constants())
    ulps = np.abs(y.cpu().numpy().view(np.int32).astype(np.int64) - model.view(np.int32))
    assert ulps.max() <= 1
