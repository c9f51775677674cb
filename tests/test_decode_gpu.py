"""GPU parity of the paged single-token decode (attn_decode_paged) against the
fp64 oracle, through the C ABI, on seeded synthetic page pools.

Covers lengths at and around page and chunk boundaries (0, 1, 15, 16, 17,
511, 512, 513, ...), MHA / GQA / MQA head sharing, both head dims, placement
invariance (the same tokens on other pages give bit-identical results), the
autoregressive check against the causal prefill, a corrupt block table (status
bit in the call's own workspace and NaN outputs, no out-of-range access), two
concurrent decodes on two streams that each report only their own status, and
the full-size workload (every sequence) in the launch configuration bench.py
times.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
import exact_io_aware_101_b200 as ea
from exact_io_aware_101_b200 import synthetic as syn
from parity_helpers import assert_bf16_parity, f32

pytestmark = pytest.mark.gpu
DEV = "cuda"


def bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def make_case(lens, Hq, Hkv, d, num_pages, max_blocks, seed):
    cfg = syn.Decode(name="case", S=len(lens), Hq=Hq, Hkv=Hkv, d=d, num_pages=num_pages,
                     max_blocks=max_blocks, seed=seed)
    return cfg, syn.decode_inputs(cfg, device="cpu", seq_lens=lens)


def oracle_decode(inp, scale, seq_ids=None):
    return oracle.decode_paged(inp["q"].float().numpy(), bits(inp["k_pages"]),
                               bits(inp["v_pages"]), inp["block_table"].numpy(),
                               inp["seq_lens"].numpy(), scale=scale, seq_ids=seq_ids)


def gpu_decode(inp, scale, workspace=None):
    d = {k: v.to(DEV) for k, v in inp.items()}
    o, l = ea.attn_decode_paged(d["q"], d["k_pages"], d["v_pages"], d["block_table"],
                                d["seq_lens"], scale=scale, workspace=workspace)
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
    ([1025, 96], 32, 1, 64),        # MQA with 32 query heads
    ([250, 17, 48], 6, 2, 128),     # group of 3
    ([700, 33], 32, 16, 128),       # 16 K/V heads: two groups of 8 per CTA grid
    ([400, 1500], 32, 2, 128),      # group of 16: two chunks of 8 query heads
]


@pytest.mark.parametrize("lens,Hq,Hkv,d", CASES)
def test_decode_small(lens, Hq, Hkv, d):
    max_blocks = max(1, max(-(-n // 16) for n in lens)) + 3
    cfg, inp = make_case(lens, Hq, Hkv, d, num_pages=sum(-(-n // 16) for n in lens) + 20,
                         max_blocks=max_blocks, seed=len(lens) + Hq + d)
    o_ref, l_ref = oracle_decode(inp, cfg.scale)
    o, l = gpu_decode(inp, cfg.scale)
    assert_bf16_parity(o, l, o_ref, l_ref, (lens, Hq, Hkv, d))
    assert ea.device_status() == 0


def test_decode_zero_length():
    cfg, inp = make_case([0, 20, 0], 8, 2, 128, num_pages=10, max_blocks=4, seed=3)
    o, l = gpu_decode(inp, cfg.scale)
    of, lf = f32(o), f32(l)
    assert np.all(of[0] == 0) and np.all(of[2] == 0)
    assert np.all(np.isneginf(lf[0])) and np.all(np.isneginf(lf[2]))
    o_ref, l_ref = oracle_decode(inp, cfg.scale, seq_ids=[1])
    assert_bf16_parity(o[1:2], l[1:2], o_ref, l_ref)


def test_decode_placement_invariance_bitwise():
    lens = [700, 33, 1500]
    cfg, inp = make_case(lens, 8, 2, 128, num_pages=200, max_blocks=100, seed=9)
    o1, l1 = gpu_decode(inp, cfg.scale)
    # Move every sequence's pages to other page ids (same tokens, same order).
    P = inp["k_pages"].shape[0]
    perm = torch.randperm(P, generator=torch.Generator().manual_seed(1)).to(torch.int32)
    bt2 = inp["block_table"].clone()
    kp2, vp2 = torch.zeros_like(inp["k_pages"]), torch.zeros_like(inp["v_pages"])
    used = bt2 >= 0
    bt2[used] = perm[inp["block_table"][used].long()]
    kp2[perm.long()] = inp["k_pages"]
    vp2[perm.long()] = inp["v_pages"]
    inp2 = dict(inp, k_pages=kp2, v_pages=vp2, block_table=bt2)
    o2, l2 = gpu_decode(inp2, cfg.scale)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_decode_matches_causal_prefill_rows():
    # Autoregressive check (Phase 08 page, Lab 01 "How to Test"): the decode of
    # token t against the cache of tokens 0..t is row t of the causal prefill.
    H, Hkv, N, d = 8, 2, 300, 128
    q, k, v = syn.random_qkv(1, H, Hkv, N, d, seed=21)
    o_pf, l_pf = ea.attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), causal=True)
    ts = [0, 15, 16, 17, 127, 128, 299]
    npg = -(-N // 16)
    kp = torch.zeros(npg, Hkv, 16, d, dtype=torch.bfloat16)
    vp = torch.zeros_like(kp)
    for t in range(N):
        kp[t // 16, :, t % 16] = k[0, :, t]
        vp[t // 16, :, t % 16] = v[0, :, t]
    bt = torch.arange(npg, dtype=torch.int32)[None].repeat(len(ts), 1).contiguous()
    lens = torch.tensor([t + 1 for t in ts], dtype=torch.int32)
    qd = torch.stack([q[0, :, t] for t in ts]).contiguous()
    inp = dict(q=qd, k_pages=kp, v_pages=vp, block_table=bt, seq_lens=lens)
    o, l = gpu_decode(inp, 1.0 / math.sqrt(d))
    for i, t in enumerate(ts):
        assert (o[i].float() - o_pf[0, :, t].float()).abs().max().item() <= 2e-2
        assert (l[i] - l_pf[0, :, t]).abs().max().item() <= 5e-3


def test_decode_bad_page_sets_status_and_nan():
    cfg, inp = make_case([40, 40], 8, 2, 128, num_pages=12, max_blocks=4, seed=5)
    good_bt = inp["block_table"]
    bt = good_bt.clone()
    bt[1, 1] = 12          # one past the pool: must not be dereferenced
    inp = dict(inp, block_table=bt)
    assert ea.device_status(clear=True) == 0
    ws = workspace_for(inp)
    o, l = gpu_decode(inp, cfg.scale, workspace=ws)
    # The call's own status word holds the bit; the per-device word stays clear.
    assert ea.decode_read_status(ws) == ea.ATTN_DEV_BAD_PAGE
    assert ea.device_status() == 0
    assert torch.isnan(o[1].float()).all() and torch.isnan(l[1]).all()
    o_ref, l_ref = oracle_decode(inp, cfg.scale, seq_ids=[0])
    assert_bf16_parity(o[0:1], l[0:1], o_ref, l_ref)
    # The next call on the same workspace clears the word it inherited.
    o2, l2 = gpu_decode(dict(inp, block_table=good_bt), cfg.scale, workspace=ws)
    assert ea.decode_read_status(ws) == 0
    assert torch.isfinite(o2.float()).all() and torch.isfinite(l2).all()


def test_decode_bad_length_sets_status():
    # A length past max_blocks * 16 is caught on the device too (the table
    # cannot hold it); the other sequence is unaffected.
    cfg, inp = make_case([40, 40], 8, 2, 128, num_pages=12, max_blocks=4, seed=6)
    inp = dict(inp, seq_lens=torch.tensor([40, 4 * 16 + 1], dtype=torch.int32))
    ws = workspace_for(inp)
    o, l = gpu_decode(inp, cfg.scale, workspace=ws)
    assert ea.decode_read_status(ws) == ea.ATTN_DEV_BAD_PAGE
    assert torch.isnan(o[1].float()).all() and torch.isnan(l[1]).all()
    o_ref, l_ref = oracle_decode(inp, cfg.scale, seq_ids=[0])
    assert_bf16_parity(o[0:1], l[0:1], o_ref, l_ref)


def test_decode_status_is_per_call_on_two_streams():
    # Two decodes run concurrently on two streams with their own workspaces;
    # only the one whose block table is corrupt reports ATTN_DEV_BAD_PAGE, and
    # neither touches the per-device word.
    cfg, inp = make_case([900, 40, 3000], 8, 2, 128, num_pages=300, max_blocks=200, seed=8)
    bad_bt = inp["block_table"].clone()
    bad_bt[2, 150] = -7
    dev_good = {k: v.to(DEV) for k, v in inp.items()}
    dev_bad = dict(dev_good, block_table=bad_bt.to(DEV))
    ws_good, ws_bad = workspace_for(inp), workspace_for(inp)
    assert ea.device_status(clear=True) == 0
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    outs = {}
    for name, st, dv, ws in (("good", s1, dev_good, ws_good), ("bad", s2, dev_bad, ws_bad)):
        with torch.cuda.stream(st):
            outs[name] = ea.attn_decode_paged(dv["q"], dv["k_pages"], dv["v_pages"],
                                              dv["block_table"], dv["seq_lens"],
                                              scale=cfg.scale, workspace=ws)
    s1.synchronize()
    assert ea.decode_read_status(ws_good) == 0
    s2.synchronize()
    assert ea.decode_read_status(ws_bad) == ea.ATTN_DEV_BAD_PAGE
    assert ea.device_status() == 0
    o_ref, l_ref = oracle_decode(inp, cfg.scale)
    assert_bf16_parity(outs["good"][0], outs["good"][1], o_ref, l_ref, "good stream")
    ob, lb = outs["bad"]
    assert torch.isnan(ob[2].float()).all() and torch.isnan(lb[2]).all()
    assert_bf16_parity(ob[:2], lb[:2], o_ref[:2], l_ref[:2], "bad stream, good sequences")


def test_decode_full_size_workload():
    cfg = syn.DECODE
    inp = syn.decode_inputs(cfg, device=DEV)
    ws = workspace_for(inp)
    o, l = ea.attn_decode_paged(inp["q"], inp["k_pages"], inp["v_pages"], inp["block_table"],
                                inp["seq_lens"], scale=cfg.scale, workspace=ws)
    torch.cuda.synchronize()
    assert ea.decode_read_status(ws) == 0 and ea.device_status() == 0
    assert torch.isfinite(o.float()).all() and torch.isfinite(l).all()
    # Compare every sequence (all heads) with the oracle; gather only the pages
    # they use so the host copy holds no unused page.
    seqs = list(range(cfg.S))
    bt = inp["block_table"][seqs]
    used = torch.unique(bt[bt >= 0])
    remap = torch.full((cfg.num_pages,), -1, dtype=torch.int32, device=DEV)
    remap[used.long()] = torch.arange(used.numel(), dtype=torch.int32, device=DEV)
    bt_small = torch.where(bt >= 0, remap[bt.clamp(min=0).long()], bt)
    small = dict(q=inp["q"][seqs].cpu(), k_pages=inp["k_pages"][used.long()].cpu(),
                 v_pages=inp["v_pages"][used.long()].cpu(), block_table=bt_small.cpu(),
                 seq_lens=inp["seq_lens"][seqs].cpu())
    o_ref, l_ref = oracle_decode(small, cfg.scale)
    assert_bf16_parity(o[seqs], l[seqs], o_ref, l_ref, "decode full size")
