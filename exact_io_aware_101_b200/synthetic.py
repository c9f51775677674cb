"""Seeded synthetic workloads for exact attention (inputs only, no attention math).

The pages measure on synthetic data only (Phase 08 page, Lab 01 "Datasets":
Synthetic), so every input here is i.i.d. N(0, 1) from a seeded torch
generator, cast to bf16 where the workload is bf16.  Both the CUDA path and the
CPU oracle take their inputs from these functions; nothing here computes any
part of attention.

Workloads (sizes of the Lab 01 benchmark sweep, seq_len 512..8192, and of the
causal, grouped-query and paged-decode extensions):

* ``TINY``    fp32, B=1, H=1, N=128, d=64, non-causal           seed 0
* ``MHA``     bf16, B=2, H=16, d=128, N in {512..8192}, non-causal seed 1000+N
* ``CAUSAL``  bf16, B=1, H=32, N=8192, d=128, causal             seed 2
* ``GQA``     bf16, B=4, Hq=32, Hkv=8, N=4096, d=128, causal     seed 3
* ``DECODE``  bf16 paged decode, 64 sequences, Hq=32, Hkv=8, d=128,
  lengths uniform in [512, 8192], 16-token pages from a 40000-page pool placed
  by a random permutation                                        seed 4
  The 8-bit cache variants (E4M3, INT8) quantise the same pools per
  (page, K/V head) slice with scale = amax / qmax (quantize_pages).
* ``CHUNKED`` chunked prefill over a paged cache: 16 sequences, a 512-token
  chunk each after ctx ~ U[0, 7680] cached tokens, Hq=32, Hkv=8, d=128,
  16-token pages placed by a random permutation                  seed 7

Generation order for a prefill workload: q, k, v from one generator.  For the
decode workload: seq_lens (randint, CPU), the page permutation (randperm, CPU),
then q, k_pages, v_pages from a generator on ``device`` seeded the same way.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Prefill:
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    causal: bool
    dtype: str  # "bf16" or "f32"
    seed: int
    window: int = 0      # sliding window (with causal): keys with i - j >= window masked
    alibi: bool = False  # ALiBi bias with the geometric slopes of alibi_slopes(Hq)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def flops(self) -> float:
        """Algorithmic FLOPs: 4*d per visible (query, key) pair -- 4*B*Hq*N^2*d,
        halved when causal (the workloads' convention), fewer with a window."""
        if self.window > 0:
            n, w = self.N, min(self.window, self.N)
            pairs = w * (w + 1) / 2.0 + (n - w) * w
            return 4.0 * self.B * self.Hq * pairs * self.d
        f = 4.0 * self.B * self.Hq * self.N * self.N * self.d
        return f / 2.0 if self.causal else f

    @property
    def bytes(self) -> int:
        """Algorithmic HBM bytes: read Q, K, V once, write O and L once."""
        es = 2 if self.dtype == "bf16" else 4
        qo = self.B * self.Hq * self.N * self.d * es
        kv = self.B * self.Hkv * self.N * self.d * es
        return 2 * qo + 2 * kv + self.B * self.Hq * self.N * 4


@dataclass(frozen=True)
class Decode:
    name: str = "decode_paged_gqa"
    S: int = 64
    Hq: int = 32
    Hkv: int = 8
    d: int = 128
    page_size: int = 16
    num_pages: int = 40000
    max_blocks: int = 512
    ctx_lo: int = 512
    ctx_hi: int = 8192
    seed: int = 4

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


TINY = Prefill("tiny_fp32", 1, 1, 1, 128, 64, False, "f32", 0)
MHA_SWEEP = tuple(Prefill("mha_n%d" % n, 2, 16, 16, n, 128, False, "bf16", 1000 + n)
                  for n in (512, 1024, 2048, 4096, 8192))
CAUSAL = Prefill("causal_n8192", 1, 32, 32, 8192, 128, True, "bf16", 2)
GQA = Prefill("gqa_causal_n4096", 4, 32, 8, 4096, 128, True, "bf16", 3)
DECODE = Decode()
# Lab 01 extensions: a Mistral-style window of 4096 keys and ALiBi, both causal,
# on the causal workload's shape.
WINDOW = Prefill("window4096_causal_n8192", 1, 32, 32, 8192, 128, True, "bf16", 5, window=4096)
ALIBI = Prefill("alibi_causal_n8192", 1, 32, 32, 8192, 128, True, "bf16", 6, alibi=True)


def alibi_slopes(H: int) -> list:
    """The geometric ALiBi slopes 2^(-8 (h+1) / H), h = 0..H-1 (Press et al.)."""
    return [2.0 ** (-8.0 * (h + 1) / H) for h in range(H)]


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def prefill_inputs(cfg: Prefill, device="cpu"):
    """(q, k, v): q [B,Hq,N,d], k/v [B,Hkv,N,d], N(0,1) values in cfg.dtype."""
    g = _gen(device, cfg.seed)
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    q = torch.randn(cfg.B, cfg.Hq, cfg.N, cfg.d, generator=g, device=device).to(dt)
    k = torch.randn(cfg.B, cfg.Hkv, cfg.N, cfg.d, generator=g, device=device).to(dt)
    v = torch.randn(cfg.B, cfg.Hkv, cfg.N, cfg.d, generator=g, device=device).to(dt)
    return q, k, v


def random_qkv(B, Hq, Hkv, N, d, seed, dtype=torch.bfloat16, device="cpu"):
    """Ad-hoc shapes for parity and edge cases, same recipe as the workloads."""
    g = _gen(device, seed)
    q = torch.randn(B, Hq, N, d, generator=g, device=device).to(dtype)
    k = torch.randn(B, Hkv, N, d, generator=g, device=device).to(dtype)
    v = torch.randn(B, Hkv, N, d, generator=g, device=device).to(dtype)
    return q, k, v


def page_placement(seq_lens, num_pages: int, max_blocks: int, page_size: int, seed: int):
    """Block table from a seeded permutation of the page pool.

    Sequence s takes the next ceil(len_s / page_size) page ids of the permutation,
    in order; unused entries are -1.  Raises if the pool is too small.
    """
    g = _gen("cpu", seed + 7919)
    perm = torch.randperm(num_pages, generator=g).to(torch.int32)
    S = len(seq_lens)
    table = torch.full((S, max_blocks), -1, dtype=torch.int32)
    nxt = 0
    for s in range(S):
        n = (int(seq_lens[s]) + page_size - 1) // page_size
        if n > max_blocks or nxt + n > num_pages:
            raise ValueError("page pool or block table too small for the lengths")
        table[s, :n] = perm[nxt:nxt + n]
        nxt += n
    return table


def decode_inputs(cfg: Decode = DECODE, device="cpu", seq_lens=None):
    """dict(q [S,Hq,d], k_pages/v_pages [P,Hkv,16,d] bf16, block_table, seq_lens)."""
    gc = _gen("cpu", cfg.seed)
    if seq_lens is None:
        seq_lens = torch.randint(cfg.ctx_lo, cfg.ctx_hi + 1, (cfg.S,), generator=gc,
                                 dtype=torch.int64).to(torch.int32)
    else:
        seq_lens = torch.as_tensor(seq_lens, dtype=torch.int32)
    table = page_placement(seq_lens, cfg.num_pages, cfg.max_blocks, cfg.page_size, cfg.seed)
    g = _gen(device, cfg.seed)
    q = torch.randn(cfg.S, cfg.Hq, cfg.d, generator=g, device=device).to(torch.bfloat16)
    shape = (cfg.num_pages, cfg.Hkv, cfg.page_size, cfg.d)
    k_pages = torch.randn(shape, generator=g, device=device).to(torch.bfloat16)
    v_pages = torch.randn(shape, generator=g, device=device).to(torch.bfloat16)
    return dict(q=q, k_pages=k_pages, v_pages=v_pages,
                block_table=table.to(device), seq_lens=seq_lens.to(device))


@dataclass(frozen=True)
class Chunked:
    """Chunked prefill over a paged cache: S sequences, each with a chunk of
    qlen new tokens after ctx cached ones, ctx uniform in [ctx_lo, ctx_hi]."""
    name: str = "chunked_prefill_gqa"
    S: int = 16
    qlen: int = 512
    Hq: int = 32
    Hkv: int = 8
    d: int = 128
    page_size: int = 16
    ctx_lo: int = 0
    ctx_hi: int = 7680
    max_blocks: int = 512
    seed: int = 7

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


CHUNKED = Chunked()


def chunked_inputs(cfg: Chunked = CHUNKED, device="cpu", qlens=None, ctxs=None, num_pages=None):
    """dict(q [T,Hq,d] bf16 token-major, k_pages/v_pages [P,Hkv,16,d] bf16,
    block_table [S,max_blocks], seq_lens [S] (= ctx + qlen), cu_q [S+1]).

    Generation order: ctx (randint, CPU), the page permutation, then q,
    k_pages, v_pages from a generator on ``device``.  The pool holds exactly the
    pages the sequences use plus 16 spare ones."""
    gc = _gen("cpu", cfg.seed)
    S = cfg.S if qlens is None else len(qlens)
    if ctxs is None:
        ctxs = torch.randint(cfg.ctx_lo, cfg.ctx_hi + 1, (S,), generator=gc, dtype=torch.int64)
    ctxs = torch.as_tensor(ctxs, dtype=torch.int64)
    qlens = torch.full((S,), cfg.qlen, dtype=torch.int64) if qlens is None else \
        torch.as_tensor(qlens, dtype=torch.int64)
    seq_lens = (ctxs + qlens).to(torch.int32)
    if num_pages is None:
        num_pages = int(sum((int(n) + cfg.page_size - 1) // cfg.page_size for n in seq_lens)) + 16
    table = page_placement(seq_lens, num_pages, cfg.max_blocks, cfg.page_size, cfg.seed)
    cu_q = torch.zeros(S + 1, dtype=torch.int32)
    cu_q[1:] = torch.cumsum(qlens, 0).to(torch.int32)
    T = int(cu_q[-1])
    g = _gen(device, cfg.seed)
    q = torch.randn(T, cfg.Hq, cfg.d, generator=g, device=device).to(torch.bfloat16)
    shape = (num_pages, cfg.Hkv, cfg.page_size, cfg.d)
    k_pages = torch.randn(shape, generator=g, device=device).to(torch.bfloat16)
    v_pages = torch.randn(shape, generator=g, device=device).to(torch.bfloat16)
    return dict(q=q, k_pages=k_pages, v_pages=v_pages, block_table=table.to(device),
                seq_lens=seq_lens.to(device), cu_q=cu_q.to(device))


def chunked_flops(seq_lens, cu_q, Hq: int, d: int) -> float:
    """4*d per visible (query, key) pair: chunk query t of sequence s sees
    ctx_s + t + 1 keys."""
    total = 0
    lens = [int(x) for x in seq_lens]
    cq = [int(x) for x in cu_q]
    for s, n in enumerate(lens):
        ql = cq[s + 1] - cq[s]
        ctx = n - ql
        total += ql * ctx + ql * (ql + 1) // 2
    return 4.0 * d * Hq * total


def decode_bytes(seq_lens, Hkv: int, d: int, Hq: int, page_size: int = 16,
                 kv_elem_bytes: int = 2) -> int:
    """Algorithmic HBM bytes of one decode call.

    K and V of every visible token (kv_elem_bytes per element: 2 for bf16, 1 for
    an 8-bit cache), q and o (bf16), L (fp32) and the block-table entries the
    call follows.  A partly filled last page counts only its visible tokens.
    An 8-bit cache adds its two fp32 scales per (visited page, K/V head).
    """
    lens = [int(x) for x in seq_lens]
    kv = sum(lens) * Hkv * d * 2 * kv_elem_bytes
    S = len(lens)
    qo = 2 * S * Hq * d * 2
    lse = S * Hq * 4
    pages = sum((n + page_size - 1) // page_size for n in lens)
    bt = 4 * pages
    scales = 2 * 4 * pages * Hkv if kv_elem_bytes == 1 else 0
    return kv + qo + lse + bt + scales


# Largest code magnitude of each 8-bit cache format.
KV_QMAX = {"e4m3": 448.0, "int8": 127.0}


def quantize_pages(pages: torch.Tensor, fmt: str, chunk: int = 4096):
    """8-bit codes and per-(page, K/V head) fp32 scales for a page pool.

    pages [P, Hkv, page_size, d] (any float dtype).  scale = amax / qmax over the
    slice (1 for an all-zero slice); codes = x / scale rounded to the format
    (E4M3 by torch's float8_e4m3fn conversion, INT8 by round-half-even and a
    clamp to [-127, 127]).  This is how the synthetic cache is written; the
    decode only reads it.  Returns (codes, scales) with codes of dtype
    float8_e4m3fn or int8.
    """
    P, Hkv = pages.shape[0], pages.shape[1]
    out_dtype = torch.float8_e4m3fn if fmt == "e4m3" else torch.int8
    codes = torch.empty(pages.shape, dtype=out_dtype, device=pages.device)
    scales = torch.empty((P, Hkv), dtype=torch.float32, device=pages.device)
    for p0 in range(0, P, chunk):
        x = pages[p0:p0 + chunk].float()
        amax = x.abs().amax(dim=(2, 3))
        sc = torch.where(amax > 0, amax / KV_QMAX[fmt], torch.ones_like(amax))
        y = x / sc[:, :, None, None]
        if fmt == "e4m3":
            codes[p0:p0 + chunk] = y.to(torch.float8_e4m3fn)
        else:
            codes[p0:p0 + chunk] = torch.round(y).clamp(-127, 127).to(torch.int8)
        scales[p0:p0 + chunk] = sc
    return codes, scales


def decode_inputs_q8(cfg: Decode = DECODE, fmt: str = "e4m3", device="cpu", seq_lens=None):
    """decode_inputs with the K/V pools quantised to an 8-bit cache.

    dict(q, k_pages/v_pages (codes), k_scales/v_scales [P,Hkv] fp32, block_table,
    seq_lens): the same q, lengths and placement as decode_inputs(cfg).
    """
    inp = decode_inputs(cfg, device=device, seq_lens=seq_lens)
    kc, ks = quantize_pages(inp.pop("k_pages"), fmt)
    vc, vs = quantize_pages(inp.pop("v_pages"), fmt)
    inp.update(k_pages=kc, v_pages=vc, k_scales=ks, v_scales=vs)
    return inp
