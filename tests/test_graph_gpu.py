"""The library's launches inside CUDA graphs, on the GPU.

A serving loop captures its steady-state work once and replays it.  The
prefill launches its whole-pair grid and, behind it, a split grid as a
programmatic dependent launch; the decode launches its split kernel and the
combine kernel the same way; the backward launches three kernels.  Each test
captures a call into a torch CUDA graph after an eager warm-up (which also
runs the library's one-time attribute setup outside the capture), replays it,
and checks the replay against the eager call bit for bit, then refills the
captured input buffers with new data and checks a second replay against an
eager call on that data.
"""
from __future__ import annotations

import math

import pytest
import torch

import exact_io_aware_101_b200 as ea
from exact_io_aware_101_b200 import synthetic as syn

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _same(a: torch.Tensor, b: torch.Tensor) -> bool:
    if a.dtype == torch.bfloat16:
        return torch.equal(a.view(torch.int16), b.view(torch.int16))
    return torch.equal(a.view(torch.int32), b.view(torch.int32))


def _capture(fn):
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()  # warm-up on the capture stream
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


# (B, Hq, Hkv, N, causal): split CTAs only (32 pairs), and a full wave of whole
# pairs with split CTAs behind it (160 pairs: the dependent launch is taken).
@pytest.mark.parametrize("B,Hq,Hkv,N,causal", [(2, 4, 2, 1000, False), (1, 40, 8, 1000, True)])
def test_prefill_replays_bitwise(B, Hq, Hkv, N, causal):
    d = 128
    q, k, v = (t.to(DEV) for t in syn.random_qkv(B, Hq, Hkv, N, d, seed=700 + N + Hq))
    o = torch.empty_like(q)
    lse = torch.empty(B, Hq, N, dtype=torch.float32, device=DEV)
    g = _capture(lambda: ea.attn_fwd(q, k, v, causal=causal, out=o, lse=lse))
    for seed in (0, 1):
        if seed:
            q2, k2, v2 = syn.random_qkv(B, Hq, Hkv, N, d, seed=800 + N + Hq)
            q.copy_(q2)
            k.copy_(k2)
            v.copy_(v2)
        o.fill_(float("nan"))
        lse.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        o_e, l_e = ea.attn_fwd(q, k, v, causal=causal)
        torch.cuda.synchronize()
        assert _same(o, o_e) and _same(lse, l_e)
    assert ea.device_status() == 0


def test_decode_replays_bitwise_and_reports_in_the_workspace():
    # Lengths up to 1280 tokens: chunks of 512 with ragged last chunks.
    cfg = syn.Decode(name="graph", S=12, Hq=16, Hkv=4, d=128, num_pages=1500, max_blocks=80,
                     ctx_lo=1, ctx_hi=1280, seed=71)
    inp = {kk: t.to(DEV) for kk, t in syn.decode_inputs(cfg, device="cpu").items()}
    o = torch.empty_like(inp["q"])
    lse = torch.empty(cfg.S, cfg.Hq, dtype=torch.float32, device=DEV)
    ws = torch.empty(ea.decode_workspace_bytes(cfg.S, cfg.Hq, cfg.d, cfg.max_blocks),
                     dtype=torch.uint8, device=DEV)
    call = lambda: ea.attn_decode_paged(inp["q"], inp["k_pages"], inp["v_pages"],
                                        inp["block_table"], inp["seq_lens"], scale=cfg.scale,
                                        out=o, lse=lse, workspace=ws)
    g = _capture(call)
    for rnd in (0, 1):
        if rnd:
            inp["q"].copy_(torch.randn(inp["q"].shape, generator=torch.Generator().manual_seed(5))
                           .to(torch.bfloat16))
        o.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert ea.decode_read_status(ws) == 0
        o_e, l_e = ea.attn_decode_paged(inp["q"], inp["k_pages"], inp["v_pages"],
                                        inp["block_table"], inp["seq_lens"], scale=cfg.scale)
        torch.cuda.synchronize()
        assert _same(o, o_e) and _same(lse, l_e)


def test_backward_replays_bitwise():
    B, Hq, Hkv, N, d = 1, 8, 2, 700, 128
    q, k, v = (t.to(DEV) for t in syn.random_qkv(B, Hq, Hkv, N, d, seed=901))
    o, lse = ea.attn_fwd(q, k, v, causal=True)
    do = torch.randn(q.shape, generator=torch.Generator().manual_seed(902)).to(torch.bfloat16).to(DEV)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(ea.bwd_workspace_bytes(B, Hq, N), dtype=torch.uint8, device=DEV)
    g = _capture(lambda: ea.attn_bwd(q, k, v, o, lse, do, causal=True, dq=dq, dk=dk, dv=dv,
                                     workspace=ws))
    dq.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    e = ea.attn_bwd(q, k, v, o, lse, do, causal=True)
    torch.cuda.synchronize()
    assert _same(dq, e[0]) and _same(dk, e[1]) and _same(dv, e[2])
    assert ea.device_status() == 0
    assert math.isfinite(dq.float().abs().max().item())
