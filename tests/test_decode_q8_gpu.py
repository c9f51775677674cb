"""GPU parity of the 8-bit paged decode (attn_decode_paged_q8, E4M3 and INT8
codes with per-(page, K/V head) scales) against the fp64 oracle, through the C
ABI, on seeded synthetic caches quantised with synthetic.quantize_pages.

Covers lengths at and around page and chunk boundaries, MHA / GQA / MQA and a
group of three, both head dims, zero lengths, a corrupt block table, scales
spread over many binades, very large and very small queries, NaN codes in the
unused slots of a partly filled page (must not leak) and in a visible slot
(must propagate as in the oracle), placement invariance, and the full-size
workload in the launch configuration bench.py times.  Tolerances are those of
the bf16 paths (parity_helpers).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import exact_io_aware_101_b200 as ea
from exact_io_aware_101_b200 import synthetic as syn
from parity_helpers import assert_bf16_parity, f32

pytestmark = pytest.mark.gpu
DEV = "cuda"
FMTS = ["e4m3", "int8"]


def codes_u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.uint8).numpy()


def make_case(lens, Hq, Hkv, d, num_pages, max_blocks, seed, fmt):
    cfg = syn.Decode(name="case", S=len(lens), Hq=Hq, Hkv=Hkv, d=d, num_pages=num_pages,
                     max_blocks=max_blocks, seed=seed)
    return cfg, syn.decode_inputs_q8(cfg, fmt=fmt, device="cpu", seq_lens=lens)


def oracle_q8(inp, scale, fmt, seq_ids=None):
    return oracle.decode_paged_q8(inp["q"].float().numpy(), codes_u8(inp["k_pages"]),
                                  codes_u8(inp["v_pages"]), inp["k_scales"].cpu().numpy(),
                                  inp["v_scales"].cpu().numpy(), inp["block_table"].cpu().numpy(),
                                  inp["seq_lens"].cpu().numpy(), scale=scale, fmt=fmt,
                                  seq_ids=seq_ids)


def gpu_q8(inp, scale, fmt, workspace=None):
    d = {k: v.to(DEV) for k, v in inp.items()}
    o, l = ea.attn_decode_paged_q8(d["q"], d["k_pages"], d["v_pages"], d["k_scales"],
                                   d["v_scales"], d["block_table"], d["seq_lens"],
                                   kv_format=fmt, scale=scale, workspace=workspace)
    torch.cuda.synchronize()
    return o, l


def workspace_for(inp):
    S, Hq, d = inp["q"].shape
    n = ea.decode_workspace_bytes(S, Hq, d, inp["block_table"].shape[1])
    return torch.empty(n, dtype=torch.uint8, device=DEV)


CASES = [
    # lens, Hq, Hkv, d
    ([1, 15, 16, 17, 33], 8, 2, 128),
    ([511, 512, 513, 1000, 2], 32, 8, 128),
    ([64, 700, 1], 4, 4, 64),
    ([300, 5], 8, 1, 128),          # MQA: 8 heads share one K/V head
    ([1025, 96], 32, 1, 64),        # MQA with 32 query heads (4 head chunks)
    ([250, 17, 48], 6, 2, 128),     # group of 3
    ([129, 40], 16, 8, 64),         # group of 2
    ([1023, 1024, 1025, 2049], 16, 4, 128),  # around the 1024-token chunk boundary
    ([700, 33], 32, 16, 128),       # 16 K/V heads: two groups of 8 per CTA grid
    ([400, 1500], 32, 2, 128),      # group of 16: two chunks of 8 query heads
]


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("lens,Hq,Hkv,d", CASES)
def test_q8_small(lens, Hq, Hkv, d, fmt):
    max_blocks = max(1, max(-(-n // 16) for n in lens)) + 3
    cfg, inp = make_case(lens, Hq, Hkv, d, num_pages=sum(-(-n // 16) for n in lens) + 20,
                         max_blocks=max_blocks, seed=len(lens) + Hq + d, fmt=fmt)
    o_ref, l_ref = oracle_q8(inp, cfg.scale, fmt)
    o, l = gpu_q8(inp, cfg.scale, fmt)
    assert_bf16_parity(o, l, o_ref, l_ref, (fmt, lens, Hq, Hkv, d))
    assert ea.device_status() == 0


@pytest.mark.parametrize("fmt", FMTS)
def test_q8_zero_length(fmt):
    cfg, inp = make_case([0, 20, 0], 8, 2, 128, num_pages=10, max_blocks=4, seed=3, fmt=fmt)
    o, l = gpu_q8(inp, cfg.scale, fmt)
    of, lf = f32(o), f32(l)
    assert np.all(of[0] == 0) and np.all(of[2] == 0)
    assert np.all(np.isneginf(lf[0])) and np.all(np.isneginf(lf[2]))
    o_ref, l_ref = oracle_q8(inp, cfg.scale, fmt, seq_ids=[1])
    assert_bf16_parity(o[1:2], l[1:2], o_ref, l_ref)


@pytest.mark.parametrize("fmt", FMTS)
def test_q8_bad_page_sets_status_and_nan(fmt):
    cfg, inp = make_case([40, 40], 8, 2, 128, num_pages=12, max_blocks=4, seed=5, fmt=fmt)
    bt = inp["block_table"].clone()
    bt[1, 1] = -3          # negative: must not be dereferenced (nor its scales read)
    inp = dict(inp, block_table=bt)
    assert ea.device_status(clear=True) == 0
    ws = workspace_for(inp)
    o, l = gpu_q8(inp, cfg.scale, fmt, workspace=ws)
    # Reported in the call's own workspace word, not in the per-device word.
    assert ea.decode_read_status(ws) == ea.ATTN_DEV_BAD_PAGE
    assert ea.device_status() == 0
    assert torch.isnan(o[1].float()).all() and torch.isnan(l[1]).all()
    o_ref, l_ref = oracle_q8(inp, cfg.scale, fmt, seq_ids=[0])
    assert_bf16_parity(o[0:1], l[0:1], o_ref, l_ref)


def _abs_codes(codes: torch.Tensor, fmt: str) -> torch.Tensor:
    """Codes of |value|: E4M3 with the sign bit cleared, INT8 by abs (no -128)."""
    if fmt == "e4m3":
        return (codes.view(torch.uint8) & 0x7F).view(torch.float8_e4m3fn)
    return codes.abs()


@pytest.mark.parametrize("fmt", FMTS)
def test_q8_scales_over_many_binades(fmt):
    # Scales are applied in f32 per page: multiply V's by 2^-12 .. 2^12 and K's
    # by 2^-3 .. 2^3 (independently per page and head; K's range is kept small
    # so that the scores stay of the order of ten) and the result still matches.
    # With V spread over 24 binades and mixed signs, O is a sum of terms that
    # cancel, so the error is measured against the terms' magnitude
    # sum_t p_t |v_t| (the oracle run on |V|), the scale the f16 / bf16
    # roundings act on: |dO| <= 2e-2 * sum_t p_t |v_t| element-wise.
    cfg, inp = make_case([700, 260, 31], 16, 4, 128, num_pages=80, max_blocks=50, seed=8,
                         fmt=fmt)
    g = torch.Generator().manual_seed(11)
    P, Hkv = inp["k_scales"].shape
    kmul = 2.0 ** torch.randint(-3, 4, (P, Hkv), generator=g).float()
    vmul = 2.0 ** torch.randint(-12, 13, (P, Hkv), generator=g).float()
    inp = dict(inp, k_scales=inp["k_scales"] * kmul, v_scales=inp["v_scales"] * vmul)
    o_ref, l_ref = oracle_q8(inp, cfg.scale, fmt)
    mag, _ = oracle_q8(dict(inp, v_pages=_abs_codes(inp["v_pages"], fmt)), cfg.scale, fmt)
    o, l = gpu_q8(inp, cfg.scale, fmt)
    of = f32(o).astype(np.float64)
    assert np.all(np.isfinite(of))
    ratio = np.abs(of - o_ref) / (2e-2 * mag + 1e-30)
    assert ratio.max() <= 1.0, (fmt, float(ratio.max()))
    assert np.max(np.abs(f32(l) - l_ref)) <= 5e-3


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("qmul", [2.0 ** 12, 2.0 ** -14])
def test_q8_query_magnitudes(fmt, qmul):
    # The query is normalised per head by a power of two before it is rounded
    # to f16: huge and tiny queries keep their precision.  The softmax scale is
    # divided by the same factor so the scores stay comparable.
    cfg, inp = make_case([300, 77], 8, 2, 128, num_pages=30, max_blocks=20, seed=12, fmt=fmt)
    inp = dict(inp, q=(inp["q"].float() * qmul).to(torch.bfloat16))
    scale = cfg.scale / qmul
    o_ref, l_ref = oracle_q8(inp, scale, fmt)
    o, l = gpu_q8(inp, scale, fmt)
    assert_bf16_parity(o, l, o_ref, l_ref, (fmt, qmul))


def test_q8_nan_codes_in_unused_slots_do_not_leak():
    # Slots past a sequence's end in its last page are never part of the
    # result: fill them with E4M3 NaN codes and nothing changes, bit for bit.
    fmt = "e4m3"
    lens = [37, 5, 16]
    cfg, inp = make_case(lens, 8, 2, 128, num_pages=12, max_blocks=4, seed=13, fmt=fmt)
    o1, l1 = gpu_q8(inp, cfg.scale, fmt)
    kb = inp["k_pages"].view(torch.uint8).clone()
    vb = inp["v_pages"].view(torch.uint8).clone()
    for s, n in enumerate(lens):
        if n % 16:
            p = int(inp["block_table"][s, n // 16])
            kb[p, :, n % 16:] = 0x7F
            vb[p, :, n % 16:] = 0xFF
    inp2 = dict(inp, k_pages=kb.view(torch.float8_e4m3fn), v_pages=vb.view(torch.float8_e4m3fn))
    o2, l2 = gpu_q8(inp2, cfg.scale, fmt)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert torch.isfinite(o1.float()).all()


def test_q8_nan_code_in_visible_slot_propagates():
    # A NaN code among a sequence's visible keys makes the attention of every
    # query head of that K/V head NaN, in the oracle and on the GPU alike.
    fmt = "e4m3"
    cfg, inp = make_case([40, 40], 8, 2, 128, num_pages=10, max_blocks=4, seed=14, fmt=fmt)
    kb = inp["k_pages"].view(torch.uint8).clone()
    p = int(inp["block_table"][0, 1])
    kb[p, 1, 3, 7] = 0x7F     # sequence 0, K/V head 1, token 19
    inp = dict(inp, k_pages=kb.view(torch.float8_e4m3fn))
    o_ref, l_ref = oracle_q8(inp, cfg.scale, fmt)
    o, l = gpu_q8(inp, cfg.scale, fmt)
    of, lf = f32(o), f32(l)
    np.testing.assert_array_equal(np.isnan(of), np.isnan(o_ref))
    np.testing.assert_array_equal(np.isnan(lf), np.isnan(l_ref))
    assert np.isnan(of[0, 4:8]).all() and not np.isnan(of[0, 0:4]).any()
    assert_bf16_parity(o[1:2], l[1:2], o_ref[1:2], l_ref[1:2])


@pytest.mark.parametrize("fmt", FMTS)
def test_q8_placement_invariance_bitwise(fmt):
    lens = [700, 33, 1500]
    cfg, inp = make_case(lens, 8, 2, 128, num_pages=200, max_blocks=100, seed=9, fmt=fmt)
    o1, l1 = gpu_q8(inp, cfg.scale, fmt)
    P = inp["k_pages"].shape[0]
    perm = torch.randperm(P, generator=torch.Generator().manual_seed(1)).to(torch.int32)
    bt2 = inp["block_table"].clone()
    used = bt2 >= 0
    bt2[used] = perm[inp["block_table"][used].long()]
    kp2 = torch.zeros_like(inp["k_pages"].view(torch.uint8))
    vp2 = torch.zeros_like(kp2)
    kp2[perm.long()] = inp["k_pages"].view(torch.uint8)
    vp2[perm.long()] = inp["v_pages"].view(torch.uint8)
    ks2 = torch.zeros_like(inp["k_scales"])
    vs2 = torch.zeros_like(inp["v_scales"])
    ks2[perm.long()] = inp["k_scales"]
    vs2[perm.long()] = inp["v_scales"]
    dt = inp["k_pages"].dtype
    inp2 = dict(inp, k_pages=kp2.view(dt), v_pages=vp2.view(dt), k_scales=ks2, v_scales=vs2,
                block_table=bt2)
    o2, l2 = gpu_q8(inp2, cfg.scale, fmt)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_q8_e4m3_as_uint8_bytes_is_identical():
    cfg, inp = make_case([200, 9], 8, 2, 128, num_pages=20, max_blocks=16, seed=15, fmt="e4m3")
    o1, l1 = gpu_q8(inp, cfg.scale, "e4m3")
    inp2 = dict(inp, k_pages=inp["k_pages"].view(torch.uint8),
                v_pages=inp["v_pages"].view(torch.uint8))
    o2, l2 = gpu_q8(inp2, cfg.scale, "e4m3")
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("fmt", FMTS)
def test_q8_full_size_workload(fmt):
    cfg = syn.DECODE
    inp = syn.decode_inputs_q8(cfg, fmt=fmt, device=DEV)
    ws = workspace_for(inp)
    o, l = ea.attn_decode_paged_q8(inp["q"], inp["k_pages"], inp["v_pages"], inp["k_scales"],
                                   inp["v_scales"], inp["block_table"], inp["seq_lens"],
                                   kv_format=fmt, scale=cfg.scale, workspace=ws)
    torch.cuda.synchronize()
    assert ea.decode_read_status(ws) == 0 and ea.device_status() == 0
    assert torch.isfinite(o.float()).all() and torch.isfinite(l).all()
    seqs = list(range(cfg.S))  # every sequence
    bt = inp["block_table"][seqs]
    used = torch.unique(bt[bt >= 0])
    remap = torch.full((cfg.num_pages,), -1, dtype=torch.int32, device=DEV)
    remap[used.long()] = torch.arange(used.numel(), dtype=torch.int32, device=DEV)
    bt_small = torch.where(bt >= 0, remap[bt.clamp(min=0).long()], bt)
    small = dict(q=inp["q"][seqs].cpu(), k_pages=inp["k_pages"][used.long()].cpu(),
                 v_pages=inp["v_pages"][used.long()].cpu(),
                 k_scales=inp["k_scales"][used.long()].cpu(),
                 v_scales=inp["v_scales"][used.long()].cpu(), block_table=bt_small.cpu(),
                 seq_lens=inp["seq_lens"][seqs].cpu())
    o_ref, l_ref = oracle_q8(small, cfg.scale, fmt)
    assert_bf16_parity(o[seqs], l[seqs], o_ref, l_ref, "q8 decode full size " + fmt)
