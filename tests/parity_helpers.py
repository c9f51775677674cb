"""Shared tolerances and comparison helpers for the GPU parity tests.

Tolerances (element-wise, against the fp64 oracle on the same inputs):
  * float32 path: max |dO| <= 1e-4 (the Lab 01 bar of the Phase 08 page:
    "within 1e-4" of standard attention);
  * bf16 paths: max |dO| <= 2e-2, mean |dO| <= 2e-3, max |dL| <= 5e-3.
    O is rounded to bf16 (relative step 2^-8, so |O| <~ 4 gives up to ~8e-3
    from the final rounding alone) and P is fed to the second GEMM in bf16.
"""
import numpy as np
import torch

F32_MAX_O = 1e-4
BF16_MAX_O = 2e-2
BF16_MEAN_O = 2e-3
BF16_MAX_L = 5e-3


def f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def errors(o_gpu, l_gpu, o_ref, l_ref):
    o = f32(o_gpu).astype(np.float64)
    l = f32(l_gpu).astype(np.float64)
    do = np.abs(o - o_ref)
    dl = np.abs(l - l_ref)
    return dict(max_o=float(do.max()) if do.size else 0.0,
                mean_o=float(do.mean()) if do.size else 0.0,
                max_l=float(dl.max()) if dl.size else 0.0)


def assert_bf16_parity(o_gpu, l_gpu, o_ref, l_ref, what=""):
    e = errors(o_gpu, l_gpu, o_ref, l_ref)
    assert np.isfinite(f32(o_gpu)).all() and np.isfinite(f32(l_gpu)).all(), what
    assert e["max_o"] <= BF16_MAX_O, (what, e)
    assert e["mean_o"] <= BF16_MEAN_O, (what, e)
    assert e["max_l"] <= BF16_MAX_L, (what, e)
    return e


def assert_f32_parity(o_gpu, l_gpu, o_ref, l_ref, what=""):
    e = errors(o_gpu, l_gpu, o_ref, l_ref)
    assert e["max_o"] <= F32_MAX_O, (what, e)
    assert e["max_l"] <= F32_MAX_O, (what, e)
    return e
