"""GPU parity of the prefill paths (attn_fwd bf16, attn_fwd_f32) against the
fp64 oracle, through the C ABI, on seeded synthetic inputs.

Small shapes are compared element by element over every output; they span
several 128-row tiles, ragged tails, single rows, both head dims, causal and
not, and MHA / GQA / MQA head sharing.  The full-size workloads run in the
same launch configuration as bench.py and are compared on sampled rows the
oracle evaluates one by one, plus properties that hold at any size.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
import exact_io_aware_101_b200 as ea
from exact_io_aware_101_b200 import synthetic as syn
from parity_helpers import assert_bf16_parity, assert_f32_parity, f32

pytestmark = pytest.mark.gpu
DEV = "cuda"

SMALL = [
    # B, Hq, Hkv, N, d, causal
    (1, 1, 1, 1, 64, False),
    (1, 1, 1, 1, 128, True),
    (1, 2, 2, 17, 128, False),
    (1, 2, 2, 17, 128, True),
    (2, 4, 1, 127, 64, True),      # MQA
    (1, 4, 2, 128, 128, False),
    (1, 4, 2, 129, 128, True),
    (2, 8, 2, 255, 128, True),     # GQA, ragged second tile
    (1, 2, 2, 256, 64, False),
    (1, 2, 1, 257, 128, True),
    (1, 3, 1, 384, 128, False),    # last CTA holds one valid Q tile
    (1, 2, 2, 1000, 128, False),
    (1, 2, 2, 1000, 128, True),
    (1, 2, 2, 1000, 64, True),
    (1, 1, 1, 2048, 128, True),    # many causal tile pairs
    (3, 6, 3, 640, 128, True),
]


def run_small(B, Hq, Hkv, N, d, causal, seed):
    q, k, v = syn.random_qkv(B, Hq, Hkv, N, d, seed=seed)
    scale = 1.0 / math.sqrt(d)
    o_ref, l_ref = oracle.attention(q.float().numpy(), k.float().numpy(), v.float().numpy(),
                                    scale=scale, causal=causal)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    out = torch.full_like(qd, float("nan"))   # poison: every row must be written
    lse = torch.full((B, Hq, N), float("nan"), device=DEV)
    o, l = ea.attn_fwd(qd, kd, vd, causal=causal, scale=scale, out=out, lse=lse)
    torch.cuda.synchronize()
    return o, l, o_ref, l_ref


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal", SMALL)
def test_bf16_small_shapes(B, Hq, Hkv, N, d, causal):
    o, l, o_ref, l_ref = run_small(B, Hq, Hkv, N, d, causal, seed=100 + N + d + Hq)
    assert_bf16_parity(o, l, o_ref, l_ref, (B, Hq, Hkv, N, d, causal))
    assert ea.device_status() == 0


# Which grid a launch uses depends on its count of 256-row Q-tile pairs
# (B * Hq * ceil(N / 256)) against the SM count: pairs that do not fill the
# last wave, when they are at most half the SMs and no window is set, run as
# two split CTAs each (one Q tile, its KV range halved over the two softmax
# warpgroups) in a second grid behind the whole pairs.  The SMALL shapes above
# all have at most 74 pairs, so on a 148-SM part they run split CTAs only.
# These shapes reach the other two cases: whole pairs only, and a full wave of
# whole pairs plus split CTAs for the rest.
GRID_CASES = [
    # label, B, Hq, Hkv, N, d, causal, alibi
    ("whole", 1, 24, 6, 1100, 128, True, False),     # GQA, ragged last tile
    ("whole", 2, 12, 1, 900, 64, False, False),      # MQA, d = 64
    ("mixed", 1, 40, 8, 1000, 128, True, False),     # GQA causal
    ("mixed", 1, 32, 32, 1200, 128, True, True),     # ALiBi causal
    ("mixed", 2, 16, 4, 1280, 64, False, False),     # d = 64 non-causal
]


def grid_kind(B, Hq, N, sms, window=0):
    pairs = B * Hq * ((N + 255) // 256)
    rem = pairs % sms
    split = window == 0 and rem > 0 and 2 * rem <= sms
    if not split:
        return "whole"
    return "split" if pairs < sms else "mixed"


@pytest.mark.parametrize("label,B,Hq,Hkv,N,d,causal,alibi", GRID_CASES)
def test_bf16_whole_and_mixed_grids(label, B, Hq, Hkv, N, d, causal, alibi):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    if grid_kind(B, Hq, N, sms) != label:
        pytest.skip("this shape takes another grid on a %d-SM device" % sms)
    q, k, v = syn.random_qkv(B, Hq, Hkv, N, d, seed=500 + N + d + Hq)
    scale = 1.0 / math.sqrt(d)
    sl = slopes_for(Hq) if alibi else None
    o_ref, l_ref = oracle.attention(q.float().numpy(), k.float().numpy(), v.float().numpy(),
                                    scale=scale, causal=causal,
                                    alibi_slopes=None if sl is None else sl.numpy())
    out = torch.full_like(q, float("nan"), device=DEV)
    lse = torch.full((B, Hq, N), float("nan"), device=DEV)
    o, l = ea.attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), causal=causal, scale=scale, out=out,
                       lse=lse, alibi_slopes=None if sl is None else sl.to(DEV))
    torch.cuda.synchronize()
    assert_bf16_parity(o, l, o_ref, l_ref, (label, B, Hq, Hkv, N, d, causal, alibi))
    assert ea.device_status() == 0


def test_grid_kinds_of_the_shapes():
    # On a 148-SM B200 every GRID_CASES shape takes the grid its label names,
    # and the SMALL shapes take split CTAs only.
    for label, B, Hq, _, N, _, _, _ in GRID_CASES:
        assert grid_kind(B, Hq, N, 148) == label
    for B, Hq, _, N, _, _ in SMALL:
        assert grid_kind(B, Hq, N, 148) == "split"


def test_bf16_deterministic_and_gqa_equals_repeated_heads():
    B, Hq, Hkv, N, d = 2, 8, 2, 700, 128
    q, k, v = (t.to(DEV) for t in syn.random_qkv(B, Hq, Hkv, N, d, seed=7))
    o1, l1 = ea.attn_fwd(q, k, v, causal=True)
    o2, l2 = ea.attn_fwd(q, k, v, causal=True)
    G = Hq // Hkv
    o3, l3 = ea.attn_fwd(q, k.repeat_interleave(G, 1).contiguous(),
                         v.repeat_interleave(G, 1).contiguous(), causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert torch.equal(o1, o3) and torch.equal(l1, l3)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("d", [64, 128])
def test_bf16_large_scores_stay_finite(causal, d):
    # Scores of several hundred: only the running-max shift keeps exp finite, and
    # exponents far below -126 reach the exp2 of unmasked tiles.
    B, H, N = 1, 2, 300
    q, k, v = syn.random_qkv(B, H, H, N, d, seed=11)
    q = (q.float() * 8).to(torch.bfloat16)
    o_ref, l_ref = oracle.attention(q.float().numpy(), k.float().numpy(), v.float().numpy(),
                                    scale=1.0, causal=causal)
    o, l = ea.attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), causal=causal, scale=1.0)
    torch.cuda.synchronize()
    assert np.abs(l_ref).max() > 100
    # L is large in magnitude here; hold it to the same absolute bound relative to |L|.
    e = np.abs(f32(l) - l_ref) / np.maximum(1.0, np.abs(l_ref))
    assert e.max() <= 5e-3
    assert np.abs(f32(o) - o_ref).max() <= 2e-2


# An unmasked tile after the first may compute P against the running max
# before it looks for the tile's own max, and keeps that P only when every
# row's sum stays at most 255.  One key here scores far above every earlier
# key for every query (all queries positive, that key constant): its x = s*c - m
# lands within 8 (the P stands), across 8 for some rows only, near 50, or near
# 200 (where 2^x overflows fp32), at several columns of the tile.  A row that
# misses must fall back to the max-first step; every case must match the oracle.
@pytest.mark.parametrize("col,a,causal", [(46, 16.0, False), (46, 16.0, True), (46, 4.0, False),
                                          (46, 0.75, False), (40, 16.0, False), (47, 1.0, True)])
def test_bf16_score_jump_after_the_first_tile(col, a, causal):
    B, H, N, d = 1, 2, 640, 128
    g = torch.Generator().manual_seed(1234)
    q = torch.randn(B, H, N, d, generator=g).abs().to(torch.bfloat16)
    k = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    J = 256 + col  # third KV tile
    k[:, :, J, :] = a
    scale = 1.0 / math.sqrt(d)
    o_ref, l_ref = oracle.attention(q.float().numpy(), k.float().numpy(), v.float().numpy(),
                                    scale=scale, causal=causal)
    o, l = ea.attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), causal=causal, scale=scale)
    torch.cuda.synchronize()
    # The jump in log2 units over the best earlier key, for the rows that see J.
    s = np.einsum("bhnd,bhkd->bhnk", q.double().numpy(), k.double().numpy()) * scale / math.log(2)
    jump = s[:, :, J:, J] - s[:, :, J:, :J].max(-1)
    assert jump.min() > {16.0: 150, 4.0: 30, 1.0: 5, 0.75: 2}[a]
    # l_ref is near a * sum(q) * scale for rows past J: compare relative to |L|.
    e = np.abs(f32(l) - l_ref) / np.maximum(1.0, np.abs(l_ref))
    assert e.max() <= 5e-3
    assert np.abs(f32(o) - o_ref).max() <= 2e-2
    assert ea.device_status() == 0


# ALiBi, on the whole-pair grid (74 heads x 2 pairs = one full wave): such a
# CTA walks its KV tiles from the last down, so the bias falls along the walk
# and an unmasked tile may keep P against the running max.  One key of the
# first KV tile (the last one walked) scores far above the rest for every
# query, so the P of that tile must be dropped and the tile redone max first,
# with the bias added again to the scores it reads back.
@pytest.mark.parametrize("col,a,causal", [(46, 16.0, True), (46, 4.0, False), (100, 0.75, True)])
def test_bf16_alibi_score_jump_whole_pairs(col, a, causal):
    B, H, N, d = 1, 74, 512, 128
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    if grid_kind(B, H, N, sms) != "whole":
        pytest.skip("this shape takes another grid on a %d-SM device" % sms)
    g = torch.Generator().manual_seed(2468)
    q = torch.randn(B, H, N, d, generator=g).abs().to(torch.bfloat16)
    k = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    k[:, :, col, :] = a
    scale = 1.0 / math.sqrt(d)
    sl = slopes_for(H)
    o_ref, l_ref = oracle.attention(q.float().numpy(), k.float().numpy(), v.float().numpy(),
                                    scale=scale, causal=causal, alibi_slopes=sl.numpy())
    o, l = ea.attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), causal=causal, scale=scale,
                       alibi_slopes=sl.to(DEV))
    torch.cuda.synchronize()
    e = np.abs(f32(l) - l_ref) / np.maximum(1.0, np.abs(l_ref))
    assert e.max() <= 5e-3
    assert np.abs(f32(o) - o_ref).max() <= 2e-2
    assert ea.device_status() == 0


def test_bf16_score_jump_inside_a_window():
    # As above, under a 300-key causal window: the jump sits in the window of
    # the later rows only, and rows whose window starts in a masked first tile
    # keep a reference max that a later tile may exceed.
    B, H, N, d = 1, 2, 1000, 128
    g = torch.Generator().manual_seed(4321)
    q = torch.randn(B, H, N, d, generator=g).abs().to(torch.bfloat16)
    k = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    k[:, :, 520, :] = 4.0
    scale = 1.0 / math.sqrt(d)
    o_ref, l_ref = oracle.attention(q.float().numpy(), k.float().numpy(), v.float().numpy(),
                                    scale=scale, causal=True, window=300)
    o, l = ea.attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), causal=True, scale=scale, window=300)
    torch.cuda.synchronize()
    e = np.abs(f32(l) - l_ref) / np.maximum(1.0, np.abs(l_ref))
    assert e.max() <= 5e-3
    assert np.abs(f32(o) - o_ref).max() <= 2e-2
    assert ea.device_status() == 0


def test_fp32_tiny_workload():
    cfg = syn.TINY
    q, k, v = syn.prefill_inputs(cfg)
    o_ref, l_ref = oracle.attention(q.numpy(), k.numpy(), v.numpy(), scale=cfg.scale)
    o, l = ea.attn_fwd_f32(q.to(DEV), k.to(DEV), v.to(DEV), scale=cfg.scale)
    torch.cuda.synchronize()
    assert_f32_parity(o, l, o_ref, l_ref, cfg.name)


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal", [
    (1, 1, 1, 1, 64, False), (1, 2, 1, 33, 128, True), (2, 4, 2, 200, 64, True),
    (1, 2, 2, 513, 128, False), (1, 8, 1, 100, 128, False)])
def test_fp32_shapes(B, Hq, Hkv, N, d, causal):
    q, k, v = syn.random_qkv(B, Hq, Hkv, N, d, seed=5 + N, dtype=torch.float32)
    o_ref, l_ref = oracle.attention(q.numpy(), k.numpy(), v.numpy(), scale=0.1, causal=causal)
    o, l = ea.attn_fwd_f32(q.to(DEV), k.to(DEV), v.to(DEV), causal=causal, scale=0.1)
    torch.cuda.synchronize()
    assert_f32_parity(o, l, o_ref, l_ref, (B, Hq, Hkv, N, d, causal))


def sample_rows(B, Hq, N, n_random, seed):
    """Flat row indices: tile-edge and random rows of random heads, plus every
    row of the last (batch, head) -- a whole head covers every Q-tile position
    of the grid's last CTAs."""
    rng = np.random.default_rng(seed)
    fixed = [0, 1, 127, 128, 129, 255, 256, N // 2, N - 129, N - 128, N - 2, N - 1]
    rows = []
    for r in fixed:
        if 0 <= r < N:
            rows.append((int(rng.integers(B)), int(rng.integers(Hq)), r))
    for _ in range(n_random):
        rows.append((int(rng.integers(B)), int(rng.integers(Hq)), int(rng.integers(N))))
    rows += [(B - 1, Hq - 1, i) for i in range(N)]
    return np.unique(np.array([(b * Hq + h) * N + i for b, h, i in rows], dtype=np.int64))


def full_size_check(cfg, n_random=64):
    q, k, v = syn.prefill_inputs(cfg, device=DEV)
    o, l = ea.attn_fwd(q, k, v, causal=cfg.causal, scale=cfg.scale)
    torch.cuda.synchronize()
    assert ea.device_status() == 0
    # properties at any size: finite, and each output column inside the range of
    # the values it averages (a convex combination of rows of V).
    assert torch.isfinite(o.float()).all() and torch.isfinite(l).all()
    G = cfg.Hq // cfg.Hkv
    vmin = v.float().amin(dim=2).repeat_interleave(G, 1)[:, :, None, :]
    vmax = v.float().amax(dim=2).repeat_interleave(G, 1)[:, :, None, :]
    of = o.float()
    assert bool((of >= vmin - 1e-2).all()) and bool((of <= vmax + 1e-2).all())
    rows = sample_rows(cfg.B, cfg.Hq, cfg.N, n_random, cfg.seed)
    qh, kh, vh = q.float().cpu().numpy(), k.float().cpu().numpy(), v.float().cpu().numpy()
    o_ref, l_ref = oracle.attention_rows(qh, kh, vh, cfg.scale, cfg.causal, rows)
    o_s = o.reshape(-1, cfg.d)[torch.from_numpy(rows).to(DEV)]
    l_s = l.reshape(-1)[torch.from_numpy(rows).to(DEV)]
    return assert_bf16_parity(o_s, l_s, o_ref, l_ref, cfg.name)


@pytest.mark.parametrize("cfg", syn.MHA_SWEEP, ids=lambda c: c.name)
def test_full_size_mha(cfg):
    full_size_check(cfg)


@pytest.mark.parametrize("cfg", [syn.CAUSAL, syn.GQA], ids=lambda c: c.name)
def test_full_size_causal_and_gqa(cfg):
    full_size_check(cfg)


# ------------------------------------------------ sliding window and ALiBi

EXT_SMALL = [
    # B, Hq, Hkv, N, d, window, alibi
    (1, 2, 2, 300, 128, 1, False),
    (1, 2, 1, 300, 128, 17, True),
    (1, 4, 2, 513, 128, 128, False),
    (2, 2, 2, 700, 64, 200, True),
    (1, 2, 2, 1000, 128, 129, False),
    (1, 2, 2, 1000, 128, 0, True),
    (1, 2, 2, 640, 128, 5000, True),   # window wider than the sequence
    (1, 8, 2, 900, 128, 300, True),    # GQA
]


def slopes_for(Hq):
    return torch.tensor(syn.alibi_slopes(Hq), dtype=torch.float32)


@pytest.mark.parametrize("B,Hq,Hkv,N,d,window,alibi", EXT_SMALL)
def test_bf16_window_alibi_small(B, Hq, Hkv, N, d, window, alibi):
    q, k, v = syn.random_qkv(B, Hq, Hkv, N, d, seed=300 + N + window)
    scale = 1.0 / math.sqrt(d)
    sl = slopes_for(Hq) if alibi else None
    o_ref, l_ref = oracle.attention(q.float().numpy(), k.float().numpy(), v.float().numpy(),
                                    scale=scale, causal=True, window=window,
                                    alibi_slopes=None if sl is None else sl.numpy())
    out = torch.full_like(q, float("nan"), device=DEV)
    lse = torch.full((B, Hq, N), float("nan"), device=DEV)
    o, l = ea.attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), causal=True, scale=scale, out=out,
                       lse=lse, window=window, alibi_slopes=None if sl is None else sl.to(DEV))
    torch.cuda.synchronize()
    assert_bf16_parity(o, l, o_ref, l_ref, (B, Hq, Hkv, N, d, window, alibi))
    assert ea.device_status() == 0


@pytest.mark.parametrize("window,alibi", [(1, False), (37, True), (200, False), (0, True)])
def test_fp32_window_alibi(window, alibi):
    B, Hq, Hkv, N, d = 1, 4, 2, 260, 64
    q, k, v = syn.random_qkv(B, Hq, Hkv, N, d, seed=40 + window, dtype=torch.float32)
    sl = slopes_for(Hq) if alibi else None
    o_ref, l_ref = oracle.attention(q.numpy(), k.numpy(), v.numpy(), scale=0.125, causal=True,
                                    window=window, alibi_slopes=None if sl is None else sl.numpy())
    o, l = ea.attn_fwd_f32(q.to(DEV), k.to(DEV), v.to(DEV), causal=True, scale=0.125,
                           window=window, alibi_slopes=None if sl is None else sl.to(DEV))
    torch.cuda.synchronize()
    assert_f32_parity(o, l, o_ref, l_ref, (window, alibi))


def test_window_wider_than_sequence_equals_causal_bitwise():
    q, k, v = (t.to(DEV) for t in syn.random_qkv(1, 4, 2, 777, 128, seed=9))
    o1, l1 = ea.attn_fwd(q, k, v, causal=True)
    o2, l2 = ea.attn_fwd(q, k, v, causal=True, window=777)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("cfg", [syn.WINDOW, syn.ALIBI], ids=lambda c: c.name)
def test_full_size_window_and_alibi(cfg):
    q, k, v = syn.prefill_inputs(cfg, device=DEV)
    sl = slopes_for(cfg.Hq).to(DEV) if cfg.alibi else None
    o, l = ea.attn_fwd(q, k, v, causal=True, scale=cfg.scale, window=cfg.window, alibi_slopes=sl)
    torch.cuda.synchronize()
    assert ea.device_status() == 0
    assert torch.isfinite(o.float()).all() and torch.isfinite(l).all()
    rows = sample_rows(cfg.B, cfg.Hq, cfg.N, 64, cfg.seed)
    o_ref, l_ref = oracle.attention_rows(q.float().cpu().numpy(), k.float().cpu().numpy(),
                                         v.float().cpu().numpy(), cfg.scale, True, rows,
                                         window=cfg.window,
                                         alibi_slopes=None if sl is None else sl.cpu().numpy())
    idx = torch.from_numpy(rows).to(DEV)
    assert_bf16_parity(o.reshape(-1, cfg.d)[idx], l.reshape(-1)[idx], o_ref, l_ref, cfg.name)
