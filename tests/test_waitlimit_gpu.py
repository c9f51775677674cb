"""Bounded waits that run out: the abort path of the kernels, on the GPU.

Every wait in the library's kernels gives up after a cycle limit, raises
ATTN_DEV_TIMEOUT, lets the copies and MMAs already in flight land, frees tensor
memory and returns -- it never traps or hangs.  In the product build the limit is
about 1.5 s and no legitimate wait comes near it, so these tests use a separate
build of the same sources (exact_io_aware_101_b200.build.build_test_lib):
waits limited to about 1 ms, and producers that stop before ring index 2 without
arriving on its barrier or issuing its copy.  Nothing is then in flight when the
consumers' waits run out; the failure is a flag that nothing sets, not a fault.

Each test checks that the call returns, that the status bit is set where the
entry point reports it, and that the product library then computes a correct
result on the same device (the context stays usable).
"""
from __future__ import annotations

import ctypes
import math

import numpy as np
import pytest
import torch

import exact_io_aware_101_b200 as ea
import oracle
from exact_io_aware_101_b200 import build as eabuild
from exact_io_aware_101_b200 import synthetic as syn
from parity_helpers import assert_bf16_parity

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def tlib():
    return ea.load_library(eabuild.build_test_lib())


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _dev_status(lib, clear=True):
    st = ctypes.c_uint(0)
    assert lib.attn_device_status(ctypes.byref(st), int(clear), _stream()) == 0
    return st.value


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def test_prefill_wait_runs_out_and_the_device_stays_usable(tlib):
    # N = 512: four K/V tiles, so the producer's stop before the second K tile
    # leaves the MMA thread and both softmax warpgroups waiting.
    B, H, N, d = 1, 2, 512, 128
    q, k, v = syn.random_qkv(B, H, H, N, d, seed=40)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    o = torch.empty_like(qd)
    lse = torch.empty(B, H, N, dtype=torch.float32, device=DEV)
    assert _dev_status(tlib) == 0
    rc = tlib.attn_fwd(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), o.data_ptr(), lse.data_ptr(),
                       B, H, H, N, d, 1.0 / math.sqrt(d), 0, _stream())
    assert rc == 0
    torch.cuda.synchronize()  # the kernel returned: no hang, no fault
    assert _dev_status(tlib) == ea.ATTN_DEV_TIMEOUT
    # Same device, product library, right after: correct and no status bit.
    o2, l2 = ea.attn_fwd(qd, kd, vd)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.attention(q.float().numpy(), k.float().numpy(), v.float().numpy(),
                                    scale=1.0 / math.sqrt(d), causal=False)
    assert_bf16_parity(o2, l2, o_ref, l_ref, "product prefill after a timeout")
    assert ea.device_status() == 0


def _decode_case():
    # Sequence 0 has two pages (the producer never reaches ring index 2); the
    # others have chunks of 7, 32 and 12 pages, each stopped at its third page.
    cfg = syn.Decode(name="waitlimit", S=3, Hq=8, Hkv=2, d=128, num_pages=80, max_blocks=48,
                     seed=41)
    return cfg, syn.decode_inputs(cfg, device="cpu", seq_lens=[20, 100, 700])


def _workspace(cfg):
    n = ea.decode_workspace_bytes(cfg.S, cfg.Hq, cfg.d, cfg.max_blocks)
    return torch.empty(n, dtype=torch.uint8, device=DEV)


def _read_ws_status(lib, ws):
    st = ctypes.c_uint(0)
    assert lib.attn_decode_read_status(ws.data_ptr(), ctypes.byref(st)) == 0
    return st.value


def test_decode_wait_runs_out_and_reports_in_the_workspace(tlib):
    cfg, inp = _decode_case()
    dv = {kk: t.to(DEV) for kk, t in inp.items()}
    o = torch.empty_like(dv["q"])
    lse = torch.empty(cfg.S, cfg.Hq, dtype=torch.float32, device=DEV)
    ws = _workspace(cfg)
    assert _dev_status(tlib) == 0
    rc = tlib.attn_decode_paged(dv["q"].data_ptr(), dv["k_pages"].data_ptr(),
                                dv["v_pages"].data_ptr(), dv["block_table"].data_ptr(),
                                dv["seq_lens"].data_ptr(), o.data_ptr(), lse.data_ptr(), cfg.S,
                                cfg.Hq, cfg.Hkv, cfg.d, 16, cfg.max_blocks, cfg.num_pages,
                                cfg.scale, ws.data_ptr(), ws.numel(), _stream())
    assert rc == 0
    torch.cuda.synchronize()
    assert _read_ws_status(tlib, ws) == ea.ATTN_DEV_TIMEOUT
    assert _dev_status(tlib) == 0  # the workspace decode reports only in its workspace
    assert torch.isnan(o[1:].float()).all() and torch.isnan(lse[1:]).all()
    o_ref, l_ref = oracle.decode_paged(inp["q"].float().numpy(), _bits(inp["k_pages"]),
                                       _bits(inp["v_pages"]), inp["block_table"].numpy(),
                                       inp["seq_lens"].numpy(), scale=cfg.scale)
    assert_bf16_parity(o[:1], lse[:1], o_ref[:1], l_ref[:1], "sequence the stop never reached")
    # The product decode on the same device and workspace, right after.
    o2, l2 = ea.attn_decode_paged(dv["q"], dv["k_pages"], dv["v_pages"], dv["block_table"],
                                  dv["seq_lens"], scale=cfg.scale, workspace=ws)
    torch.cuda.synchronize()
    assert ea.decode_read_status(ws) == 0
    assert_bf16_parity(o2, l2, o_ref, l_ref, "product decode after a timeout")


def test_q8_decode_wait_runs_out_and_reports_in_the_workspace(tlib):
    cfg, _ = _decode_case()
    inp = syn.decode_inputs_q8(cfg, fmt="e4m3", device="cpu", seq_lens=[20, 100, 700])
    dv = {kk: t.to(DEV) for kk, t in inp.items()}
    o = torch.empty_like(dv["q"])
    lse = torch.empty(cfg.S, cfg.Hq, dtype=torch.float32, device=DEV)
    ws = _workspace(cfg)
    rc = tlib.attn_decode_paged_q8(dv["q"].data_ptr(), dv["k_pages"].data_ptr(),
                                   dv["v_pages"].data_ptr(), dv["k_scales"].data_ptr(),
                                   dv["v_scales"].data_ptr(), ea.KV_FORMATS["e4m3"],
                                   dv["block_table"].data_ptr(), dv["seq_lens"].data_ptr(),
                                   o.data_ptr(), lse.data_ptr(), cfg.S, cfg.Hq, cfg.Hkv, cfg.d, 16,
                                   cfg.max_blocks, cfg.num_pages, cfg.scale, ws.data_ptr(),
                                   ws.numel(), _stream())
    assert rc == 0
    torch.cuda.synchronize()
    assert _read_ws_status(tlib, ws) == ea.ATTN_DEV_TIMEOUT
    assert torch.isnan(o[1:].float()).all() and torch.isnan(lse[1:]).all()
    u8 = lambda t: t.contiguous().view(torch.uint8).numpy()
    o_ref, l_ref = oracle.decode_paged_q8(inp["q"].float().numpy(), u8(inp["k_pages"]),
                                          u8(inp["v_pages"]), inp["k_scales"].numpy(),
                                          inp["v_scales"].numpy(), inp["block_table"].numpy(),
                                          inp["seq_lens"].numpy(), scale=cfg.scale, fmt="e4m3")
    assert_bf16_parity(o[:1], lse[:1], o_ref[:1], l_ref[:1], "sequence the stop never reached")
    o2, l2 = ea.attn_decode_paged_q8(dv["q"], dv["k_pages"], dv["v_pages"], dv["k_scales"],
                                     dv["v_scales"], dv["block_table"], dv["seq_lens"],
                                     kv_format="e4m3", scale=cfg.scale, workspace=ws)
    torch.cuda.synchronize()
    assert ea.decode_read_status(ws) == 0
    assert_bf16_parity(o2, l2, o_ref, l_ref, "product q8 decode after a timeout")
