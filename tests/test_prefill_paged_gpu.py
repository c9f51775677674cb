"""GPU parity of the chunked prefill over the paged cache (attn_prefill_paged)
against the fp64 oracle, through the C ABI.

Covers chunks at the start of a sequence (ctx = 0), after short and long
contexts, chunk lengths around the 128-row Q tile and 16-token pages, one-token
chunks, empty chunks, GQA / MQA, both head dims, a sliding window and ALiBi,
page placement invariance (bit-identical), agreement with the contiguous
causal prefill when the chunk is a whole sequence, a corrupt block table and
inconsistent lengths (status bit, no out-of-range access), and the full-size
workload bench.py times on sampled sequences.
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


def bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def make(qlens, ctxs, Hq, Hkv, d, seed, max_blocks=None):
    n = [q + c for q, c in zip(qlens, ctxs)]
    mb = max_blocks or max(1, max(-(-x // 16) for x in n)) + 2
    cfg = syn.Chunked(name="case", S=len(qlens), Hq=Hq, Hkv=Hkv, d=d, max_blocks=mb, seed=seed)
    return cfg, syn.chunked_inputs(cfg, device="cpu", qlens=qlens, ctxs=ctxs)


def oracle_run(inp, scale):
    return oracle.prefill_paged(inp["q"].float().numpy(), bits(inp["k_pages"]), bits(inp["v_pages"]),
                                inp["block_table"].numpy(), inp["seq_lens"].numpy(),
                                inp["cu_q"].numpy(), scale=scale)


def gpu_run(inp, scale, max_q=None, **kw):
    d = {k: v.to(DEV) for k, v in inp.items()}
    qlens = (inp["cu_q"][1:] - inp["cu_q"][:-1]).tolist()
    mq = max(qlens) if max_q is None else max_q
    o, l = ea.attn_prefill_paged(d["q"], d["k_pages"], d["v_pages"], d["block_table"],
                                 d["seq_lens"], d["cu_q"], max_q=mq, scale=scale, **kw)
    torch.cuda.synchronize()
    return o, l


CASES = [
    # qlens, ctxs, Hq, Hkv, d
    ([100], [0], 4, 4, 128),
    ([1, 17, 128, 129], [0, 5, 300, 16], 8, 2, 128),
    ([300, 256, 40], [1000, 2, 77], 8, 8, 64),
    ([513], [700], 4, 1, 128),
    ([16, 0, 33], [15, 9, 1], 4, 2, 64),
]


@pytest.mark.parametrize("qlens,ctxs,Hq,Hkv,d", CASES)
def test_prefill_paged_small(qlens, ctxs, Hq, Hkv, d):
    cfg, inp = make(qlens, ctxs, Hq, Hkv, d, seed=sum(qlens) + d)
    o_ref, l_ref = oracle_run(inp, cfg.scale)
    o, l = gpu_run(inp, cfg.scale)
    assert_bf16_parity(o, l, o_ref, l_ref, (qlens, ctxs, Hq, Hkv, d))
    assert ea.device_status() == 0


# One cached key scores far above every earlier key for every query of its
# sequence (queries made positive, that key constant), in a KV tile after the
# first: a tile whose P against the running max sums past 255 must fall back
# to the max-first step in the paged kernel too.
@pytest.mark.parametrize("a,key", [(16.0, 300), (1.0, 700), (4.0, 1100)])
def test_prefill_paged_score_jump(a, key):
    qlens, ctxs = [200, 96], [1000, 1200]
    cfg, inp = make(qlens, ctxs, 4, 2, 128, seed=41)
    inp["q"] = inp["q"].float().abs().to(torch.bfloat16)
    for s_ in range(len(qlens)):
        pg = int(inp["block_table"][s_, key // 16])
        inp["k_pages"][pg, :, key % 16, :] = a
    o_ref, l_ref = oracle_run(inp, cfg.scale)
    o, l = gpu_run(inp, cfg.scale)
    e = np.abs(f32(l) - l_ref) / np.maximum(1.0, np.abs(l_ref))
    assert e.max() <= 5e-3
    assert np.abs(f32(o) - o_ref).max() <= 2e-2
    assert ea.device_status() == 0


@pytest.mark.parametrize("qlens,ctxs", [
    # Equal key counts (the work order breaks ties by sequence index).
    ([9, 9, 30, 9, 30], [40, 40, 19, 40, 19]),
    # More sequences than the kernel ranks (384): the grid keeps the given order.
    ([3] * 400, [i % 37 for i in range(400)]),
])
def test_prefill_paged_work_order(qlens, ctxs):
    cfg, inp = make(qlens, ctxs, 2, 1, 64, seed=len(qlens))
    o_ref, l_ref = oracle_run(inp, cfg.scale)
    o, l = gpu_run(inp, cfg.scale)
    assert_bf16_parity(o, l, o_ref, l_ref, (len(qlens), "sequences"))
    assert ea.device_status() == 0


def test_prefill_paged_window_and_alibi():
    # Window and ALiBi measured from the chunk query's absolute position;
    # checked against rows ctx.. of the contiguous causal prefill's oracle.
    qlens, ctxs, Hq, Hkv, d = [200, 130], [500, 60], 4, 2, 128
    cfg, inp = make(qlens, ctxs, Hq, Hkv, d, seed=3)
    slopes = syn.alibi_slopes(Hq)
    o, l = gpu_run(inp, cfg.scale, window=256,
                   alibi_slopes=torch.tensor(slopes, dtype=torch.float32, device=DEV))
    kb, vb = bits(inp["k_pages"]), bits(inp["v_pages"])
    cu = inp["cu_q"].numpy()
    for s, (ql, ctx) in enumerate(zip(qlens, ctxs)):
        n = ql + ctx
        bt = inp["block_table"][s].numpy()
        kc = np.stack([kb[bt[t // 16], :, t % 16] for t in range(n)], axis=1)
        vc = np.stack([vb[bt[t // 16], :, t % 16] for t in range(n)], axis=1)
        to_f = lambda x: (x.astype(np.uint32) << 16).view(np.float32)
        qf = np.zeros((1, Hq, n, d), np.float32)
        qf[0, :, ctx:] = inp["q"][cu[s]:cu[s + 1]].float().numpy().transpose(1, 0, 2)
        rows = np.array([(h * n + ctx + t) for h in range(Hq) for t in range(ql)])
        ro, rl = oracle.attention_rows(qf, to_f(kc)[None], to_f(vc)[None], cfg.scale, True, rows,
                                       window=256, alibi_slopes=slopes)
        got_o = o[cu[s]:cu[s + 1]].transpose(0, 1).reshape(-1, d)
        got_l = l[cu[s]:cu[s + 1]].transpose(0, 1).reshape(-1)
        assert_bf16_parity(got_o, got_l, ro, rl, ("window+alibi", s))


def test_prefill_paged_whole_sequence_matches_contiguous_prefill():
    # A chunk that is the whole sequence (ctx = 0) is the causal prefill.
    N, Hq, Hkv, d = 300, 4, 2, 128
    cfg, inp = make([N], [0], Hq, Hkv, d, seed=4)
    o, l = gpu_run(inp, cfg.scale)
    bt = inp["block_table"][0]
    k = torch.stack([inp["k_pages"][bt[t // 16], :, t % 16] for t in range(N)], dim=1)[None]
    v = torch.stack([inp["v_pages"][bt[t // 16], :, t % 16] for t in range(N)], dim=1)[None]
    q = inp["q"].transpose(0, 1)[None].contiguous()
    of, lf = ea.attn_fwd(q.to(DEV), k.contiguous().to(DEV), v.contiguous().to(DEV), causal=True)
    torch.cuda.synchronize()
    assert (o.float() - of[0].transpose(0, 1).float()).abs().max().item() <= 2e-2
    assert (l - lf[0].transpose(0, 1)).abs().max().item() <= 5e-3


def test_prefill_paged_placement_invariance_bitwise():
    cfg, inp = make([300, 77], [900, 40], 8, 2, 128, seed=5)
    o1, l1 = gpu_run(inp, cfg.scale)
    P = inp["k_pages"].shape[0]
    perm = torch.randperm(P, generator=torch.Generator().manual_seed(2)).to(torch.int32)
    bt2 = inp["block_table"].clone()
    used = bt2 >= 0
    bt2[used] = perm[inp["block_table"][used].long()]
    kp2, vp2 = torch.zeros_like(inp["k_pages"]), torch.zeros_like(inp["v_pages"])
    kp2[perm.long()] = inp["k_pages"]
    vp2[perm.long()] = inp["v_pages"]
    o2, l2 = gpu_run(dict(inp, k_pages=kp2, v_pages=vp2, block_table=bt2), cfg.scale)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_prefill_paged_nan_in_unused_slots_does_not_leak():
    # Cache slots past a sequence's last token hold NaN: the result is unchanged.
    cfg, inp = make([40, 33], [3, 100], 4, 2, 128, seed=6)
    o1, l1 = gpu_run(inp, cfg.scale)
    kp, vp = inp["k_pages"].clone(), inp["v_pages"].clone()
    for s, n in enumerate(inp["seq_lens"].tolist()):
        if n % 16:
            p = int(inp["block_table"][s, n // 16])
            kp[p, :, n % 16:] = float("nan")
            vp[p, :, n % 16:] = float("nan")
    o2, l2 = gpu_run(dict(inp, k_pages=kp, v_pages=vp), cfg.scale)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert torch.isfinite(o1.float()).all()


def test_prefill_paged_bad_page_and_bad_lengths():
    cfg, inp = make([40, 40, 20], [10, 10, 5], 4, 2, 128, seed=7)
    bt = inp["block_table"].clone()
    bt[1, 1] = 10 ** 6          # outside the pool
    ea.device_status(clear=True)
    o, l = gpu_run(dict(inp, block_table=bt), cfg.scale)
    assert ea.device_status(clear=True) & ea.ATTN_DEV_BAD_PAGE
    cu = inp["cu_q"].tolist()
    assert torch.isnan(o[cu[1]:cu[2]].float()).all() and torch.isnan(l[cu[1]:cu[2]]).all()
    o_ref, l_ref = oracle_run(inp, cfg.scale)
    for s in (0, 2):
        assert_bf16_parity(o[cu[s]:cu[s + 1]], l[cu[s]:cu[s + 1]], o_ref[cu[s]:cu[s + 1]],
                           l_ref[cu[s]:cu[s + 1]], ("bad page neighbour", s))
    # A chunk longer than its sequence: skipped, flagged, neighbours intact.
    sl = inp["seq_lens"].clone()
    sl[2] = 10
    o, l = gpu_run(dict(inp, seq_lens=sl), cfg.scale)
    assert ea.device_status(clear=True) & ea.ATTN_DEV_BAD_PAGE
    assert_bf16_parity(o[cu[0]:cu[1]], l[cu[0]:cu[1]], o_ref[cu[0]:cu[1]], l_ref[cu[0]:cu[1]])
    # max_q smaller than a chunk: that chunk is skipped and flagged.
    o, l = gpu_run(inp, cfg.scale, max_q=20)
    assert ea.device_status(clear=True) & ea.ATTN_DEV_BAD_PAGE
    assert_bf16_parity(o[cu[2]:cu[3]], l[cu[2]:cu[3]], o_ref[cu[2]:cu[3]], l_ref[cu[2]:cu[3]])
    assert ea.device_status() == 0


def test_prefill_paged_full_size_workload():
    cfg = syn.CHUNKED
    inp = syn.chunked_inputs(cfg, device=DEV)
    o, l = ea.attn_prefill_paged(inp["q"], inp["k_pages"], inp["v_pages"], inp["block_table"],
                                 inp["seq_lens"], inp["cu_q"], max_q=cfg.qlen, scale=cfg.scale)
    torch.cuda.synchronize()
    assert ea.device_status() == 0
    assert torch.isfinite(o.float()).all() and torch.isfinite(l).all()
    # Sampled sequences 0, 7 and 15 (their pages gathered on the host).
    cu = inp["cu_q"].cpu().numpy()
    for s in (0, 7, 15):
        n = int(inp["seq_lens"][s])
        bt = inp["block_table"][s].cpu()
        used = bt[: -(-n // 16)].long()
        small = dict(q=inp["q"][cu[s]:cu[s + 1]].cpu(), k_pages=inp["k_pages"][used.to(DEV)].cpu(),
                     v_pages=inp["v_pages"][used.to(DEV)].cpu(),
                     block_table=torch.arange(used.numel(), dtype=torch.int32)[None],
                     seq_lens=torch.tensor([n], dtype=torch.int32),
                     cu_q=torch.tensor([0, cu[s + 1] - cu[s]], dtype=torch.int32))
        o_ref, l_ref = oracle_run(small, cfg.scale)
        assert_bf16_parity(o[cu[s]:cu[s + 1]], l[cu[s]:cu[s + 1]], o_ref, l_ref, ("full", s))
