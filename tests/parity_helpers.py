"""Shared tolerances and comparison helpers for the GPU parity tests.

Tolerances (element-wise, against the fp64 oracle on the same inputs):
  * float32 path: max |dO| <= 1e-4 (the Lab 01 bar of the Phase 08 page:
    "within 1e-4" of standard attention);
  * bf16 paths: max |dO| <= 2e-2, mean |dO| <= 2e-3, max |dL| <= 5e-3.
    O is rounded to bf16 (relative step 2^-8, so |O| <~ 4 gives up to ~8e-3
    from the final rounding alone) and P is fed to the second GEMM in bf16.
  * bf16 backward (dQ, dK, dV), element-wise, with r = RMS of the element's
    own output row (the d values of one query's dQ or one key's dK / dV) and
    t = RMS of the whole reference tensor:
        |d| <= 5e-2 * r + 5e-2 * t   for every element,  mean |d| <= 1e-2 * t.
    Derivation.  (i) Rounding of the row's own terms: an output row is a sum
    over keys (or queries) whose one factor (P, dS) is rounded to bf16
    (relative <= 2^-9), and the output is rounded to bf16 (<= 2^-9): about
    0.5 % of the row's magnitude typically, under 5 % in the tail.
    (ii) D = rowsum(dO * O) is formed from the bf16 O that the forward stores
    (the method keeps only O and L): |dD_i| <= 2^-9 sum_c |dO_ic O_ic|, which
    shifts every dS_ij by -P_ij dD_i and so dQ_i by scale * dD_i * (the
    P-weighted mean key) and dK_j by a sum of such terms.  This error is
    absolute: it does not shrink with the row's own gradient (a row whose
    terms nearly cancel keeps it), and on the tests' N(0,1) data it is a few
    percent of the tensor's RMS at most; hence the second term.  t is floored
    at 1e-4: an all-zero reference (dQ and dK at N = 1, where P = 1 and dS = 0
    exactly) keeps the fp32 difference between D and the MMA's dP, ~1e-7.
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


GRAD_MEAN = 1e-2
GRAD_MAX = 5e-2


def grad_errors(g_gpu, g_ref):
    """max: largest |d| / (GRAD_MAX * (r + t)) (<= 1 passes); mean: mean |d| / t."""
    g = f32(g_gpu).astype(np.float64)
    ref = np.asarray(g_ref, dtype=np.float64)
    dd = ref.shape[-1]
    g2, r2 = g.reshape(-1, dd), ref.reshape(-1, dd)
    if r2.size == 0:
        return dict(max=0.0, mean=0.0, where=None)
    t = max(float(np.sqrt(np.mean(r2 ** 2))), 1e-4)
    r = np.sqrt(np.mean(r2 ** 2, axis=1, keepdims=True))
    d = np.abs(g2 - r2)
    e = d / (GRAD_MAX * (r + t))
    w = np.unravel_index(int(np.argmax(e)), e.shape)
    return dict(max=float(e.max()), mean=float(d.mean()) / t, where=(int(w[0]), int(w[1])),
                row_rms=float(r[w[0], 0]), tensor_rms=t, got=float(g2[w]), ref=float(r2[w]))


def assert_grad_parity(g_gpu, g_ref, what=""):
    assert np.isfinite(f32(g_gpu)).all(), what
    e = grad_errors(g_gpu, g_ref)
    assert e["mean"] <= GRAD_MEAN and e["max"] <= 1.0, (what, e)
    return e
