"""attn_decode_paged_noalloc: the paged decode for callers that cannot allocate.

Some callers of this library may not call cudaMalloc -- a plugin whose host
program owns every byte of device memory through its own pool, or a decode loop
that must never wait on the allocator (cudaMalloc/cudaFree can block until the
device is idle).  For them the library keeps a fixed scratch array in its own
device memory and this entry point uses it in place of a caller workspace.

The GPU test calls the new entry point through the C ABI, twice in a row (the
scratch keeps the previous call's partials, which must not leak into the next
result), and checks both outputs against attn_decode_paged with a separately
allocated workspace, within the bf16 tolerances the other decode tests use.
Before the second call the scratch is filled with NaN partials from a longer
problem of the same shape, so a result that read a stale slot would show it;
the small case is also checked against the fp64 oracle.
This file is named to be collected last, so a run that stops at the first
failure has already run every other test.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import exact_io_aware_101_b200 as ea
import oracle
from exact_io_aware_101_b200 import synthetic as syn
from parity_helpers import BF16_MAX_L, BF16_MAX_O, BF16_MEAN_O, assert_bf16_parity


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _poison_scratch(lib, cfg, inp):
    """A noalloc call on NaN pages with every sequence at the longest length the
    block table allows: it leaves a NaN partial in every scratch slot that a
    problem of this shape (S, Hq, d, max_blocks) can use."""
    npg = cfg.S * cfg.max_blocks
    kp = torch.full((npg, cfg.Hkv, cfg.page_size, cfg.d), float("nan"), dtype=torch.bfloat16,
                    device="cuda")
    bt = torch.arange(npg, dtype=torch.int32, device="cuda").view(cfg.S, cfg.max_blocks)
    sl = torch.full((cfg.S,), cfg.max_blocks * cfg.page_size, dtype=torch.int32, device="cuda")
    poison = dict(q=inp["q"], k_pages=kp, v_pages=kp, block_table=bt, seq_lens=sl)
    cfg_p = syn.Decode(name="poison", S=cfg.S, Hq=cfg.Hq, Hkv=cfg.Hkv, d=cfg.d, num_pages=npg,
                       max_blocks=cfg.max_blocks, seed=0)
    o = torch.empty_like(inp["q"])
    l = torch.empty(cfg.S, cfg.Hq, dtype=torch.float32, device="cuda")
    assert _noalloc(lib, poison, cfg_p, o, l) == 0
    torch.cuda.synchronize()
    assert torch.isnan(l).all()


def _noalloc(lib, inp, cfg, o, lse):
    st = torch.cuda.current_stream().cuda_stream
    return lib.attn_decode_paged_noalloc(
        inp["q"].data_ptr(), inp["k_pages"].data_ptr(), inp["v_pages"].data_ptr(),
        inp["block_table"].data_ptr(), inp["seq_lens"].data_ptr(), o.data_ptr(), lse.data_ptr(),
        cfg.S, cfg.Hq, cfg.Hkv, cfg.d, cfg.page_size, cfg.max_blocks, cfg.num_pages, cfg.scale,
        st)


def _with_workspace(lib, inp, cfg, o, lse):
    ws_bytes = lib.attn_decode_workspace_bytes(cfg.S, cfg.Hq, cfg.d, cfg.max_blocks, cfg.page_size)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    rc = lib.attn_decode_paged(
        inp["q"].data_ptr(), inp["k_pages"].data_ptr(), inp["v_pages"].data_ptr(),
        inp["block_table"].data_ptr(), inp["seq_lens"].data_ptr(), o.data_ptr(), lse.data_ptr(),
        cfg.S, cfg.Hq, cfg.Hkv, cfg.d, cfg.page_size, cfg.max_blocks, cfg.num_pages, cfg.scale,
        ws.data_ptr(), ws_bytes, st)
    torch.cuda.synchronize()
    return rc


def _close(o, l, o_ref, l_ref):
    do = (o.float() - o_ref.float()).abs()
    assert do.max().item() <= BF16_MAX_O and do.mean().item() <= BF16_MEAN_O
    assert (l - l_ref).abs().max().item() <= BF16_MAX_L


@pytest.mark.gpu
@pytest.mark.parametrize("which", ["small", "full"])
def test_noalloc_matches_workspace_decode_twice(which):
    lib = ea.library()
    if which == "small":
        cfg = syn.Decode(name="noalloc_small", S=6, Hq=32, Hkv=8, d=128, num_pages=600,
                         max_blocks=96, seed=12)
        inp = syn.decode_inputs(cfg, device="cuda", seq_lens=[1, 16, 17, 513, 1500, 700])
    else:
        cfg = syn.DECODE
        inp = syn.decode_inputs(cfg, device="cuda")
    o_ref = torch.empty_like(inp["q"])
    l_ref = torch.empty(cfg.S, cfg.Hq, dtype=torch.float32, device="cuda")
    assert _with_workspace(lib, inp, cfg, o_ref, l_ref) == 0
    for call in range(2):
        if call == 1 and which == "small":
            _poison_scratch(lib, cfg, inp)
        o = torch.full_like(inp["q"], float("nan"))
        l = torch.full((cfg.S, cfg.Hq), float("nan"), device="cuda")
        assert _noalloc(lib, inp, cfg, o, l) == 0, call
        torch.cuda.synchronize()
        _close(o, l, o_ref, l_ref)
        if which == "small":
            host = {k: v.cpu() for k, v in inp.items()}
            o_or, l_or = oracle.decode_paged(host["q"].float().numpy(), _bits(host["k_pages"]),
                                             _bits(host["v_pages"]), host["block_table"].numpy(),
                                             host["seq_lens"].numpy(), scale=cfg.scale)
            assert_bf16_parity(o, l, o_or, l_or, "noalloc vs oracle, call %d" % call)
    assert ea.device_status() == 0


@pytest.mark.gpu
def test_noalloc_bad_page_reports_in_the_device_word():
    # The scratch (and its status word) is shared, so this entry point reports a
    # corrupt block table in the per-device word.
    lib = ea.library()
    cfg = syn.Decode(name="noalloc_bad", S=2, Hq=8, Hkv=2, d=128, num_pages=12, max_blocks=4,
                     seed=5)
    inp = syn.decode_inputs(cfg, device="cuda", seq_lens=[40, 40])
    inp["block_table"][1, 1] = 12  # one past the pool
    assert ea.device_status(clear=True) == 0
    o = torch.empty_like(inp["q"])
    l = torch.empty(cfg.S, cfg.Hq, dtype=torch.float32, device="cuda")
    assert _noalloc(lib, inp, cfg, o, l) == 0
    torch.cuda.synchronize()
    assert ea.device_status(clear=True) == ea.ATTN_DEV_BAD_PAGE
    assert torch.isnan(l[1]).all() and torch.isfinite(l[0]).all()
    assert ea.device_status() == 0


@pytest.mark.gpu
def test_noalloc_back_to_back_different_inputs():
    # Two different problems through the shared scratch: the second result must
    # not depend on what the first left behind.
    lib = ea.library()
    cfg_a = syn.Decode(name="a", S=4, Hq=8, Hkv=2, d=128, num_pages=300, max_blocks=64, seed=31)
    cfg_b = syn.Decode(name="b", S=3, Hq=8, Hkv=2, d=128, num_pages=300, max_blocks=64, seed=32)
    a = syn.decode_inputs(cfg_a, device="cuda", seq_lens=[900, 30, 512, 1])
    b = syn.decode_inputs(cfg_b, device="cuda", seq_lens=[40, 1000, 77])
    ref = []
    for cfg, inp in ((cfg_a, a), (cfg_b, b)):
        o = torch.empty_like(inp["q"])
        l = torch.empty(cfg.S, cfg.Hq, dtype=torch.float32, device="cuda")
        assert _with_workspace(lib, inp, cfg, o, l) == 0
        ref.append((o, l))
    for (cfg, inp), (o_ref, l_ref) in zip(((cfg_a, a), (cfg_b, b)), ref):
        o = torch.empty_like(inp["q"])
        l = torch.empty(cfg.S, cfg.Hq, dtype=torch.float32, device="cuda")
        assert _noalloc(lib, inp, cfg, o, l) == 0
        torch.cuda.synchronize()
        _close(o, l, o_ref, l_ref)


def test_noalloc_rejects_requests_beyond_the_scratch():
    # Checked on the host before any CUDA call, so this runs without a GPU.
    lib = ea.library()
    A = 1 << 20
    S, Hq, d, maxb = 64, 64, 128, 1024
    need = lib.attn_decode_workspace_bytes(S, Hq, d, maxb, 16)
    assert need > ea.DECODE_NOALLOC_SCRATCH_BYTES
    rc = lib.attn_decode_paged_noalloc(A, A, A, A, A, A, A, S, Hq, 8, d, 16, maxb, 100, 0.1, None)
    assert rc == 1  # ATTN_ERR_INVALID_ARG
