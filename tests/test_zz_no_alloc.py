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
This file is named to be collected last, so a run that stops at the first
failure has already run every other test.
"""
from __future__ import annotations

import ctypes

import pytest
import torch

import exact_io_aware_101_b200 as ea
from exact_io_aware_101_b200 import synthetic as syn
from parity_helpers import BF16_MAX_L, BF16_MAX_O, BF16_MEAN_O


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
        o = torch.full_like(inp["q"], float("nan"))
        l = torch.full((cfg.S, cfg.Hq), float("nan"), device="cuda")
        assert _noalloc(lib, inp, cfg, o, l) == 0, call
        torch.cuda.synchronize()
        _close(o, l, o_ref, l_ref)
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
