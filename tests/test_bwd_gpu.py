"""GPU parity of the bf16 attention backward (attn_bwd) against the fp64
oracle's gradients, through the C ABI.

The forward runs on the GPU (attn_fwd / attn_fwd_ext) to give the O and L the
backward takes; the oracle differentiates the definition from q, k, v and dO
alone.  Covers ragged N around the 64- and 128-row tiles, both head dims,
MHA / GQA / MQA, causal, sliding window and ALiBi, determinism (two calls are
bit-identical), and the full-size workload (N = 8192, B = 2, H = 16) on
sampled rows and keys.  Tolerances: parity_helpers.assert_grad_parity.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import exact_io_aware_101_b200 as ea
from exact_io_aware_101_b200 import synthetic as syn
from parity_helpers import assert_grad_parity

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run_case(B, Hq, Hkv, N, d, causal, window=0, alibi=False, seed=0):
    q, k, v = syn.random_qkv(B, Hq, Hkv, N, d, seed=seed)
    g = torch.Generator().manual_seed(seed + 1)
    do = torch.randn(B, Hq, N, d, generator=g).to(torch.bfloat16)
    scale = d ** -0.5
    slopes = syn.alibi_slopes(Hq) if alibi else None
    qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, do))
    sl = None if slopes is None else torch.tensor(slopes, dtype=torch.float32, device=DEV)
    o, lse = ea.attn_fwd(qd, kd, vd, causal=causal, window=window, alibi_slopes=sl)
    dq, dk, dv = ea.attn_bwd(qd, kd, vd, o, lse, dod, causal=causal, window=window,
                             alibi_slopes=sl)
    torch.cuda.synchronize()
    assert ea.device_status() == 0
    return (q, k, v, do, scale, slopes), (dq, dk, dv), (qd, kd, vd, o, lse, dod)


CASES = [
    # B, Hq, Hkv, N, d, causal, window, alibi
    (1, 1, 1, 1, 128, False, 0, False),
    (1, 2, 2, 17, 128, False, 0, False),
    (1, 2, 2, 64, 64, True, 0, False),
    (2, 4, 2, 130, 128, True, 0, False),
    (1, 4, 1, 300, 64, False, 0, False),
    (1, 2, 2, 513, 128, True, 0, False),
    (1, 4, 4, 256, 128, False, 0, False),
    (1, 2, 1, 390, 128, True, 100, False),
    (1, 2, 2, 300, 64, True, 0, True),
    (1, 8, 2, 1000, 128, True, 257, True),   # GQA with a window and ALiBi together
    (2, 6, 3, 700, 64, False, 0, True),      # group of 2, ALiBi without a mask
    (1, 4, 2, 257, 128, True, 64, True),
]


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal,window,alibi", CASES)
def test_bwd_small(B, Hq, Hkv, N, d, causal, window, alibi):
    (q, k, v, do, scale, slopes), (dq, dk, dv), _ = run_case(B, Hq, Hkv, N, d, causal, window,
                                                            alibi, seed=N + d + Hq)
    rq, rk, rv = oracle.attention_bwd(q.float().numpy(), k.float().numpy(), v.float().numpy(),
                                      do.float().numpy(), scale=scale, causal=causal,
                                      window=window, alibi_slopes=slopes)
    what = (B, Hq, Hkv, N, d, causal, window, alibi)
    assert_grad_parity(dq, rq, ("dQ",) + what)
    assert_grad_parity(dk, rk, ("dK",) + what)
    assert_grad_parity(dv, rv, ("dV",) + what)


def test_bwd_deterministic():
    _, (dq, dk, dv), (qd, kd, vd, o, lse, dod) = run_case(2, 4, 2, 700, 128, True, seed=5)
    for _ in range(2):
        dq2, dk2, dv2 = ea.attn_bwd(qd, kd, vd, o, lse, dod, causal=True)
        torch.cuda.synchronize()
        assert torch.equal(dq, dq2) and torch.equal(dk, dk2) and torch.equal(dv, dv2)


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_full_size_sampled(causal):
    # The bench's largest backward launch: B=2, H=16, N=8192, d=128.  Sampled
    # dQ rows (all heads' first/last rows, tile edges) and dK/dV keys of two
    # heads against the oracle's row and key evaluators.
    cfg = syn.MHA_SWEEP[-1]
    q, k, v = syn.prefill_inputs(cfg, device=DEV)
    g = torch.Generator(device=DEV).manual_seed(77)
    do = torch.randn(q.shape, generator=g, device=DEV).to(torch.bfloat16)
    o, lse = ea.attn_fwd(q, k, v, causal=causal)
    dq, dk, dv = ea.attn_bwd(q, k, v, o, lse, do, causal=causal)
    torch.cuda.synchronize()
    assert ea.device_status() == 0
    for t in (dq, dk, dv):
        assert torch.isfinite(t.float()).all()
    N, d, H = cfg.N, cfg.d, cfg.Hq
    # Only heads 0 and 17 are needed on the host.
    heads = [0, 17]
    sel = lambda t: t.reshape(-1, N, d)[heads].reshape(1, len(heads), N, d).float().cpu().numpy()
    qh, kh, vh, doh = sel(q), sel(k), sel(v), sel(do)
    rows = np.array([0, 1, 63, 64, 127, 128, 4095, 4096, 8190, 8191])
    rows2 = np.concatenate([rows, N + rows])
    ref_q = oracle.attention_bwd_dq_rows(qh, kh, vh, doh, cfg.scale, causal, rows2)
    got_q = dq.reshape(-1, N, d)[heads].reshape(-1, d)[torch.as_tensor(rows2, device=DEV)]
    assert_grad_parity(got_q, ref_q, "dQ rows")
    ref_k, ref_v = oracle.attention_bwd_dkv_rows(qh, kh, vh, doh, cfg.scale, causal, rows2)
    idx = torch.as_tensor(rows2, device=DEV)
    assert_grad_parity(dk.reshape(-1, N, d)[heads].reshape(-1, d)[idx], ref_k, "dK keys")
    assert_grad_parity(dv.reshape(-1, N, d)[heads].reshape(-1, d)[idx], ref_v, "dV keys")
