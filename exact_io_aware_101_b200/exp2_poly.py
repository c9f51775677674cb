"""Coefficients of the cubic that approximates 2^f on [0, 1).

The bf16 prefill kernel evaluates a quarter of its softmax exponentials on the
FMA pipe instead of the special-function unit, as

    2^x = 2^j * 2^f,   j = floor(x),  f = x - j in [0, 1),
    2^f ~= c0 + c1 f + c2 f^2 + c3 f^3,

adding j to the IEEE-754 exponent field of the cubic's value.  The cubic is a
near-minimax fit in relative error, found here by Lawson's iteratively
reweighted least squares on a dense grid; rounded to float32 and evaluated with
float32 Horner steps its relative error stays below 2^-13, far inside the
2^-8 relative step of the bf16 P that the second GEMM consumes.
``tests/test_exp2_poly.py`` re-runs the fit and checks the constants compiled
into ``csrc/prefill_sm100.cu`` and the error bound.
"""
from __future__ import annotations

import numpy as np


def fit(degree: int = 3, points: int = 20001, iters: int = 200):
    f = np.linspace(0.0, 1.0, points)
    y = np.exp2(f)
    V = np.vstack([f ** k for k in range(degree + 1)]).T
    w = np.ones_like(f)
    c = None
    for _ in range(iters):
        W = w / y
        c, *_ = np.linalg.lstsq(V * W[:, None], y * W, rcond=None)
        err = (V @ c - y) / y
        w = w * np.sqrt(np.abs(err)) + 1e-30
        w /= w.sum()
    return c.astype(np.float32)


def horner_f32(c, f):
    """Evaluate the cubic the way the kernel does: float32 fused multiply-adds."""
    f = np.asarray(f, dtype=np.float32)
    p = np.full_like(f, c[-1])
    for k in range(len(c) - 2, -1, -1):
        p = (p.astype(np.float64) * f + np.float64(c[k])).astype(np.float32)
    return p


def exp2_model(x, c):
    """Reference model of the kernel's full 2^x (clamp, floor split, exponent add)."""
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-126.0))
    j = np.floor(x).astype(np.int64)
    f = (x - j.astype(np.float32)).astype(np.float32)
    p = horner_f32(c, f)
    bits = p.view(np.uint32).astype(np.int64) + (j << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


if __name__ == "__main__":
    c = fit()
    print([float(v).hex() for v in c])
