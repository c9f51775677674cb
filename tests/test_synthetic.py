"""The seeded input generators and the work accounting behind the bench, on the CPU.

The roofline fractions divide these FLOP and byte counts by measured times, so
each formula is checked against a brute-force count on small shapes; the
generators are checked against the input recipe the workloads state (lengths,
page placement, chunk layout, the 8-bit cache's scales and rounding).
"""
from __future__ import annotations

import math

import pytest
import torch

from exact_io_aware_101_b200 import synthetic as syn


def _visible_pairs(N, causal, window):
    n = 0
    for i in range(N):
        for j in range(N):
            if causal and j > i:
                continue
            if window and i - j >= window:
                continue
            n += 1
    return n


@pytest.mark.parametrize("N,window", [(10, 3), (10, 10), (17, 1), (33, 16), (8, 20)])
def test_window_flops_count_every_visible_pair(N, window):
    cfg = syn.Prefill("t", 2, 3, 3, N, 64, True, "bf16", 0, window=window)
    assert cfg.flops == 4.0 * 2 * 3 * 64 * _visible_pairs(N, True, window)


def test_dense_and_causal_flops_follow_the_stated_convention():
    # 4*B*Hq*N^2*d, halved for causal (the convention of the workloads; the
    # diagonal's N extra pairs are not counted).
    dense = syn.Prefill("t", 2, 16, 16, 512, 128, False, "bf16", 0)
    causal = syn.Prefill("t", 2, 16, 16, 512, 128, True, "bf16", 0)
    assert dense.flops == 4.0 * 2 * 16 * 512 * 512 * 128
    assert causal.flops == dense.flops / 2
    assert _visible_pairs(64, False, 0) == 64 * 64
    assert abs(_visible_pairs(64, True, 0) - 64 * 64 / 2) == 32  # N/2 diagonal pairs


def test_prefill_bytes_read_inputs_once_and_write_outputs_once():
    cfg = syn.GQA
    q, k, v = (t.numel() * 2 for t in syn.random_qkv(1, cfg.Hq, cfg.Hkv, 8, cfg.d, seed=0))
    per_row = (2 * q + k + v) / 8 + cfg.Hq * 4  # q and o, k, v, one fp32 L per head
    assert cfg.bytes == cfg.B * cfg.N * per_row


def test_chunked_flops_brute_force():
    seq_lens, cu_q = [5, 9, 3], [0, 2, 6, 9]  # chunks of 2, 4, 3 after ctx 3, 5, 0
    pairs = 0
    for s, n in enumerate(seq_lens):
        ql = cu_q[s + 1] - cu_q[s]
        for t in range(ql):
            pairs += (n - ql) + t + 1  # the cached keys plus the causal part of the chunk
    assert syn.chunked_flops(seq_lens, cu_q, Hq=4, d=64) == 4.0 * 64 * 4 * pairs


@pytest.mark.parametrize("kv_bytes", [2, 1])
def test_decode_bytes_brute_force(kv_bytes):
    lens, Hkv, d, Hq = [1, 16, 17, 100], 2, 64, 8
    kv = sum(lens) * Hkv * d * 2 * kv_bytes  # K and V of every visible token
    pages = sum(math.ceil(n / 16) for n in lens)
    expect = kv + 2 * len(lens) * Hq * d * 2 + len(lens) * Hq * 4 + 4 * pages
    if kv_bytes == 1:
        expect += 2 * 4 * pages * Hkv
    assert syn.decode_bytes(lens, Hkv, d, Hq, kv_elem_bytes=kv_bytes) == expect


def test_page_placement_is_a_seeded_injection_into_the_pool():
    lens = [1, 16, 17, 250, 0]
    t = syn.page_placement(lens, num_pages=64, max_blocks=20, page_size=16, seed=3)
    assert t.dtype == torch.int32 and tuple(t.shape) == (5, 20)
    used = []
    for s, n in enumerate(lens):
        k = math.ceil(n / 16)
        assert (t[s, k:] == -1).all()
        used += t[s, :k].tolist()
    assert len(used) == len(set(used)) and all(0 <= p < 64 for p in used)
    assert torch.equal(t, syn.page_placement(lens, 64, 20, 16, seed=3))
    assert not torch.equal(t, syn.page_placement(lens, 64, 20, 16, seed=4))
    with pytest.raises(ValueError):
        syn.page_placement([400], num_pages=64, max_blocks=20, page_size=16, seed=3)
    with pytest.raises(ValueError):
        syn.page_placement([16 * 20] * 4, num_pages=64, max_blocks=20, page_size=16, seed=3)


def test_decode_workload_follows_its_recipe():
    cfg = syn.DECODE
    # The lengths and placement only (the pools of the full workload are 2.6 GB),
    # drawn as decode_inputs draws them.
    gc = torch.Generator().manual_seed(cfg.seed)
    seq_lens = torch.randint(cfg.ctx_lo, cfg.ctx_hi + 1, (cfg.S,), generator=gc)
    assert cfg.S == 64 and cfg.Hq == 32 and cfg.Hkv == 8 and cfg.d == 128
    assert cfg.page_size == 16 and cfg.num_pages == 40000
    assert int(seq_lens.min()) >= 512 and int(seq_lens.max()) <= 8192
    assert cfg.max_blocks * cfg.page_size >= 8192
    table = syn.page_placement(seq_lens, cfg.num_pages, cfg.max_blocks, cfg.page_size, cfg.seed)
    ids = table[table >= 0]
    assert ids.numel() == sum(math.ceil(int(n) / 16) for n in seq_lens)
    assert ids.unique().numel() == ids.numel()
    # A small decode through the same generator: shapes, dtypes, lengths as given.
    small = syn.Decode(name="s", S=3, Hq=8, Hkv=2, d=64, num_pages=40, max_blocks=8, seed=9)
    inp = syn.decode_inputs(small, seq_lens=[1, 100, 128])
    assert tuple(inp["q"].shape) == (3, 8, 64) and inp["q"].dtype == torch.bfloat16
    assert tuple(inp["k_pages"].shape) == (40, 2, 16, 64)
    assert inp["seq_lens"].tolist() == [1, 100, 128]
    assert (inp["block_table"][:, :8] >= -1).all()


def test_chunked_workload_layout():
    cfg = syn.Chunked(name="s", S=3, Hq=4, Hkv=2, d=64, max_blocks=16, seed=1)
    inp = syn.chunked_inputs(cfg, qlens=[5, 0, 7], ctxs=[10, 3, 0])
    assert inp["cu_q"].tolist() == [0, 5, 5, 12]
    assert inp["seq_lens"].tolist() == [15, 3, 7]
    assert tuple(inp["q"].shape) == (12, 4, 64)
    pool = inp["k_pages"].shape[0]
    assert pool == (1 + 1 + 1) + 16  # every sequence fits one page, plus 16 spare
    default = syn.CHUNKED
    assert default.S == 16 and default.qlen == 512 and (default.ctx_lo, default.ctx_hi) == (0, 7680)


@pytest.mark.parametrize("fmt", ["int8", "e4m3"])
def test_quantize_pages_scale_and_rounding(fmt):
    g = torch.Generator().manual_seed(11)
    pages = torch.randn(3, 2, 16, 64, generator=g)
    pages[1, 0] = 0.0  # an all-zero slice takes scale 1
    codes, scales = syn.quantize_pages(pages, fmt, chunk=2)  # a chunk boundary inside the pool
    qmax = syn.KV_QMAX[fmt]
    amax = pages.abs().amax(dim=(2, 3))
    assert torch.equal(scales[1, 0], torch.tensor(1.0))
    nz = amax > 0
    assert torch.allclose(scales[nz], amax[nz] / qmax, rtol=0, atol=0)
    c = codes.float()
    # The slice's largest element lands on the format's largest code.
    assert torch.equal(c.abs().amax(dim=(2, 3))[nz], torch.full_like(amax[nz], qmax))
    x = pages / scales[:, :, None, None]
    err = (c - x).abs()
    if fmt == "int8":
        assert err.max() <= 0.5 and torch.equal(c, torch.round(c))
    else:  # three mantissa bits: half a unit in the last place, 2^-4 relative (normals)
        assert (err <= x.abs() * 2.0 ** -4 + 2.0 ** -10).all()
