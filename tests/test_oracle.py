"""Pins for the fp64 CPU oracle (no GPU).

The oracle is trusted only because these checks tie it to what the pages and
the mathematics fix, independently of the oracle's own code:

* closed forms: one key (O = v0), identical keys (O = mean of V, L = s + ln N),
  constant values (weights sum to one), causal row 0, two keys (logistic weights);
* hand-derived worked examples under tests/golden/ (powers of two);
* a brute force in 50-digit decimal arithmetic, written without the max-shift
  that the oracle uses, on tiny inputs;
* the online recurrence of the Phase 08 page (Lab 01 talking points) for tile
  sizes 1, 7 and N;
* structural invariants: GQA equals MHA with repeated K/V heads, key/value
  permutation invariance, shift invariance under large offsets, causal rows
  equal non-causal attention over the prefix, paged equals contiguous;
* 8-bit KV cache: all 256 E4M3 codes against torch's float8_e4m3fn
  converter and the format's fixed points; E4M3 / INT8 decode with
  power-of-two scales equals the bf16 paged decode of the dequantised cache
  exactly; scale linearity (V's scale multiplies O, K's acts as the softmax
  scale);
* chunked prefill over the paged cache: rows ctx.. of a full causal prefill
  over the contiguous sequence; one query per chunk is the paged decode;
  splitting a chunk in two changes nothing;
* backward: gradients equal a 4-point central-difference derivative of the
  forward oracle (inputs on a 2^-10 grid so every perturbed value is exact in
  float32); the two-key closed form; invariants (dK of a head sums to zero,
  dV sums to the dO sum, constant V gives dQ = dK = 0); GQA equals MHA with
  the group's gradients summed; the sampled evaluators equal the full one;
* mutation checks: plausible one-token mistakes planted in a copy of the
  oracle's C source are each caught by at least one pin.
"""
from __future__ import annotations

import decimal
import json
import math
import os
import subprocess
import sys
from fractions import Fraction

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from oracle.online import online_attention  # noqa: E402

RNG = np.random.default_rng(12345)


def rand(*shape, rng=RNG):
    return rng.standard_normal(shape).astype(np.float32)


# ---------------------------------------------------------------- closed forms

def test_single_key_returns_its_value():
    q, k, v = rand(2, 3, 1, 8), rand(2, 3, 1, 8), rand(2, 3, 1, 8)
    o, lse = oracle.attention(q, k, v, scale=0.37)
    np.testing.assert_allclose(o, v.astype(np.float64), rtol=0, atol=1e-15)
    s = 0.37 * np.einsum("bhnd,bhnd->bhn", q.astype(np.float64), k.astype(np.float64))
    np.testing.assert_allclose(lse, s, rtol=0, atol=1e-13)


def test_identical_keys_average_the_values():
    N, d = 11, 16
    q, v = rand(1, 2, N, d), rand(1, 2, N, d)
    krow = rand(1, 2, 1, d)
    k = np.repeat(krow, N, axis=2)
    o, lse = oracle.attention(q, k, v, scale=0.25)
    mean_v = v.astype(np.float64).mean(axis=2, keepdims=True)
    np.testing.assert_allclose(o, np.broadcast_to(mean_v, o.shape), rtol=0, atol=1e-13)
    s = 0.25 * np.einsum("bhnd,bhd->bhn", q.astype(np.float64), krow[:, :, 0].astype(np.float64))
    np.testing.assert_allclose(lse, s + math.log(N), rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_weights_sum_to_one(causal):
    # With every value row equal to c, O = (sum_j p_ij) c, so O == c iff the
    # softmax weights of each row sum to one.
    N, d = 37, 8
    q, k = rand(1, 1, N, d) * 3, rand(1, 1, N, d) * 3
    c = rand(d)
    v = np.broadcast_to(c, (1, 1, N, d)).copy()
    o, _ = oracle.attention(q, k, v, scale=0.5, causal=causal)
    np.testing.assert_allclose(o, np.broadcast_to(c.astype(np.float64), o.shape), rtol=0, atol=1e-12)


def test_weights_are_nonnegative_and_normalised():
    # v_j = e_j (one-hot) exposes each row of P in O directly.
    N = 9
    q, k = rand(1, 1, N, N), rand(1, 1, N, N)  # d = N so v can be one-hot
    v = np.eye(N, dtype=np.float32)[None, None]
    for causal in (False, True):
        P, _ = oracle.attention(q, k, v, scale=1.0, causal=causal)
        P = P[0, 0]
        assert (P >= 0).all()
        np.testing.assert_allclose(P.sum(axis=1), 1.0, rtol=0, atol=1e-14)
        if causal:
            assert np.all(np.triu(P, 1) == 0.0)


def test_causal_row_zero_sees_only_key_zero():
    q, k, v = rand(1, 2, 6, 4), rand(1, 2, 6, 4), rand(1, 2, 6, 4)
    o, lse = oracle.attention(q, k, v, scale=0.7, causal=True)
    np.testing.assert_allclose(o[:, :, 0], v[:, :, 0].astype(np.float64), rtol=0, atol=1e-15)
    s00 = 0.7 * np.einsum("bhd,bhd->bh", q[:, :, 0].astype(np.float64), k[:, :, 0].astype(np.float64))
    np.testing.assert_allclose(lse[:, :, 0], s00, rtol=0, atol=1e-14)


def test_two_keys_logistic_weights():
    d = 6
    q, k, v = rand(1, 1, 1, d), rand(1, 1, 2, d), rand(1, 1, 2, d)
    o, lse = oracle.attention(q, k, v, scale=0.9)
    qd, kd, vd = q[0, 0, 0].astype(float), k[0, 0].astype(float), v[0, 0].astype(float)
    s0, s1 = 0.9 * float(qd @ kd[0]), 0.9 * float(qd @ kd[1])
    w0 = 1.0 / (1.0 + math.exp(s1 - s0))
    np.testing.assert_allclose(o[0, 0, 0], w0 * vd[0] + (1 - w0) * vd[1], rtol=0, atol=1e-14)
    hi, lo = max(s0, s1), min(s0, s1)
    np.testing.assert_allclose(lse[0, 0, 0], hi + math.log1p(math.exp(lo - hi)), rtol=0, atol=1e-14)


# ------------------------------------------------------------ golden examples

def _val(x):
    if isinstance(x, str):
        if x == "ln2":
            return math.log(2.0)
        if x.startswith("ln"):
            return math.log(float(x[2:]))
        return float(Fraction(x))
    if isinstance(x, list):
        return [_val(y) for y in x]
    return float(x)


def _golden():
    with open(os.path.join(ROOT, "tests", "golden", "hand_examples.json")) as f:
        return json.load(f)


@pytest.mark.parametrize("case", _golden()["prefill"], ids=lambda c: c["name"])
def test_golden_prefill(case):
    q, k, v = (np.array(_val(case[n]), dtype=np.float32) for n in ("q", "k", "v"))
    o, lse = oracle.attention(q, k, v, scale=_val(case["scale"]), causal=case["causal"])
    np.testing.assert_allclose(o, np.array(_val(case["o"])), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, np.array(_val(case["lse"])), rtol=0, atol=1e-12)


@pytest.mark.parametrize("case", _golden()["decode"], ids=lambda c: c["name"])
def test_golden_decode(case):
    import torch
    to_bits = lambda a: torch.tensor(a, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    kp, vp = to_bits(_val(case["k_pages"])), to_bits(_val(case["v_pages"]))
    o, lse = oracle.decode_paged(np.array(case["q"], dtype=np.float32), kp, vp,
                                 np.array(case["block_table"], dtype=np.int32),
                                 np.array(case["seq_lens"], dtype=np.int32),
                                 scale=_val(case["scale"]))
    np.testing.assert_allclose(o, np.array(_val(case["o"])), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, np.array(_val(case["lse"])), rtol=0, atol=1e-12)


# ------------------------------------------------------ decimal brute force

def _brute_decimal(q, k, v, scale, causal, G, window=0, slopes=None):
    """Per-element evaluation in 50-digit decimals: p_ij = e^{s_ij} / sum_j e^{s_ij}."""
    ctx = decimal.Context(prec=50)
    D = lambda x: ctx.create_decimal_from_float(float(x))
    B, Hq, N, d = q.shape
    o = np.zeros(q.shape)
    lse = np.zeros(q.shape[:3])
    sc = D(scale)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            for i in range(N):
                js = range(i + 1) if causal else range(k.shape[2])
                if window:
                    js = [j for j in js if i - j < window]
                e = {}
                for j in js:
                    s = ctx.multiply(sc, sum((ctx.multiply(D(q[b, h, i, c]), D(k[b, g, j, c])) for c in range(d)), decimal.Decimal(0)))
                    if slopes is not None:
                        s = s + ctx.multiply(D(slopes[h]), decimal.Decimal(j - i))
                    e[j] = ctx.exp(s)
                tot = sum(e.values(), decimal.Decimal(0))
                for c in range(d):
                    acc = sum((ctx.multiply(ctx.divide(e[j], tot), D(v[b, g, j, c])) for j in js), decimal.Decimal(0))
                    o[b, h, i, c] = float(acc)
                lse[b, h, i] = float(ctx.ln(tot))
    return o, lse


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,d,Hq,Hkv", [(1, 1, 1, 1), (3, 2, 2, 1), (5, 4, 2, 2), (8, 3, 4, 2)])
def test_decimal_brute_force(N, d, Hq, Hkv, causal):
    rng = np.random.default_rng(N * 100 + d * 10 + Hq + causal)
    q, k, v = (rng.standard_normal(s).astype(np.float32) * 2 for s in
               ((2, Hq, N, d), (2, Hkv, N, d), (2, Hkv, N, d)))
    o, lse = oracle.attention(q, k, v, scale=0.6, causal=causal)
    ob, lb = _brute_decimal(q, k, v, 0.6, causal, Hq // Hkv)
    np.testing.assert_allclose(o, ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lb, rtol=0, atol=1e-12)


@pytest.mark.parametrize("window,use_alibi", [(1, False), (2, True), (3, False), (0, True)])
def test_decimal_brute_force_window_alibi(window, use_alibi):
    rng = np.random.default_rng(window * 10 + use_alibi)
    Hq, Hkv, N, d = 4, 2, 7, 3
    q, k, v = (rng.standard_normal(s).astype(np.float32) for s in
               ((1, Hq, N, d), (1, Hkv, N, d), (1, Hkv, N, d)))
    slopes = [0.5, 0.25, 0.125, 0.0625] if use_alibi else None
    o, lse = oracle.attention(q, k, v, scale=0.6, causal=True, window=window, alibi_slopes=slopes)
    ob, lb = _brute_decimal(q, k, v, 0.6, True, Hq // Hkv, window=window, slopes=slopes)
    np.testing.assert_allclose(o, ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lb, rtol=0, atol=1e-12)


# ------------------------------------------------------- sliding window, ALiBi

def test_window_covering_everything_is_causal():
    N = 21
    q, k, v = rand(2, 4, N, 8), rand(2, 2, N, 8), rand(2, 2, N, 8)
    o1, l1 = oracle.attention(q, k, v, scale=0.3, causal=True)
    for w in (N, N + 5, 10 ** 6):
        o2, l2 = oracle.attention(q, k, v, scale=0.3, causal=True, window=w)
        np.testing.assert_array_equal(o1, o2)
        np.testing.assert_array_equal(l1, l2)


def test_window_of_one_returns_own_value():
    q, k, v = rand(1, 3, 9, 4), rand(1, 3, 9, 4), rand(1, 3, 9, 4)
    o, lse = oracle.attention(q, k, v, scale=0.45, causal=True, window=1)
    np.testing.assert_allclose(o, v.astype(np.float64), rtol=0, atol=1e-15)
    s = 0.45 * np.einsum("bhnd,bhnd->bhn", q.astype(np.float64), k.astype(np.float64))
    np.testing.assert_allclose(lse, s, rtol=0, atol=1e-13)


def test_window_rows_equal_attention_over_the_window():
    N, d, W = 14, 4, 5
    q, k, v = rand(1, 1, N, d), rand(1, 1, N, d), rand(1, 1, N, d)
    o, lse = oracle.attention(q, k, v, scale=0.8, causal=True, window=W)
    for i in range(N):
        lo = max(0, i - W + 1)
        oi, li = oracle.attention(q[:, :, i:i + 1], k[:, :, lo:i + 1], v[:, :, lo:i + 1], scale=0.8)
        np.testing.assert_array_equal(o[0, 0, i], oi[0, 0, 0])
        np.testing.assert_array_equal(lse[0, 0, i], li[0, 0, 0])


def test_alibi_zero_slopes_is_plain():
    q, k, v = rand(1, 2, 11, 8), rand(1, 2, 11, 8), rand(1, 2, 11, 8)
    for causal in (False, True):
        o1, l1 = oracle.attention(q, k, v, scale=0.2, causal=causal)
        o2, l2 = oracle.attention(q, k, v, scale=0.2, causal=causal, alibi_slopes=[0.0, 0.0])
        np.testing.assert_array_equal(o1, o2)
        np.testing.assert_array_equal(l1, l2)


@pytest.mark.parametrize("causal", [False, True])
def test_alibi_is_one_extra_dimension(causal):
    # slope_h * (j - i) = (extra coordinate slope_h of q) * (extra coordinate j of
    # k) - slope_h * i.  The last term is constant along a row, so O is that of
    # plain attention on the augmented vectors and L is lower by slope_h * i.
    B, Hq, Hkv, N, d = 1, 4, 2, 13, 5
    q, k, v = rand(B, Hq, N, d), rand(B, Hkv, N, d), rand(B, Hkv, N, d)
    slopes = np.array([0.5, 0.25, 0.125, 0.0625])
    qa = np.concatenate([q, np.broadcast_to(slopes[None, :, None, None], (B, Hq, N, 1))], axis=3)
    ka = np.concatenate([k, np.broadcast_to(np.arange(N)[None, None, :, None], (B, Hkv, N, 1))], axis=3)
    o1, l1 = oracle.attention(q, k, v, scale=1.0, causal=causal, alibi_slopes=slopes)
    # v must share d with q/k in the oracle: pad v with one zero column.
    va = np.concatenate([v, np.zeros((B, Hkv, N, 1), np.float32)], axis=3)
    o2, l2 = oracle.attention(qa.astype(np.float32), ka.astype(np.float32), va, scale=1.0, causal=causal)
    np.testing.assert_allclose(o1, o2[..., :d], rtol=0, atol=1e-12)
    shift = slopes[None, :, None] * np.arange(N)[None, None, :]
    np.testing.assert_allclose(l1, l2 - shift, rtol=0, atol=1e-11)


def test_rows_evaluator_window_alibi():
    B, Hq, Hkv, N, d = 1, 4, 2, 40, 8
    q, k, v = rand(B, Hq, N, d), rand(B, Hkv, N, d), rand(B, Hkv, N, d)
    slopes = [0.3, 0.2, 0.1, 0.05]
    o, lse = oracle.attention(q, k, v, scale=0.25, causal=True, window=9, alibi_slopes=slopes)
    rows = RNG.choice(B * Hq * N, size=30, replace=False)
    orow, lrow = oracle.attention_rows(q, k, v, 0.25, True, rows, window=9, alibi_slopes=slopes)
    np.testing.assert_allclose(orow, o.reshape(-1, d)[rows], rtol=0, atol=1e-14)
    np.testing.assert_allclose(lrow, lse.reshape(-1)[rows], rtol=0, atol=1e-14)


# ------------------------------------------------------- online recurrence

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("block", [1, 7, 64])
def test_online_recurrence_equals_two_pass(block, causal):
    N, d = 64, 16
    q, k, v = rand(1, 1, N, d) * 2, rand(1, 1, N, d) * 2, rand(1, 1, N, d)
    o, lse = oracle.attention(q, k, v, scale=0.25, causal=causal)
    oo, lo = online_attention(q[0, 0], k[0, 0], v[0, 0], 0.25, block, causal=causal)
    np.testing.assert_allclose(oo, o[0, 0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lo, lse[0, 0], rtol=0, atol=1e-12)


# -------------------------------------------------------------- invariants

def test_gqa_equals_mha_with_repeated_heads():
    B, Hq, Hkv, N, d = 2, 8, 2, 19, 8
    q, k, v = rand(B, Hq, N, d), rand(B, Hkv, N, d), rand(B, Hkv, N, d)
    for causal in (False, True):
        o1, l1 = oracle.attention(q, k, v, scale=0.3, causal=causal)
        G = Hq // Hkv
        o2, l2 = oracle.attention(q, np.repeat(k, G, axis=1), np.repeat(v, G, axis=1),
                                  scale=0.3, causal=causal)
        np.testing.assert_array_equal(o1, o2)
        np.testing.assert_array_equal(l1, l2)
    # head h uses kv head h // G (contiguous groups): head 1 must differ from
    # what kv head 1 would give.
    o_alt, _ = oracle.attention(q[:, 1:2], k[:, 1:2], v[:, 1:2], scale=0.3)
    o_ref, _ = oracle.attention(q[:, 1:2], k[:, 0:1], v[:, 0:1], scale=0.3)
    o_all, _ = oracle.attention(q, k, v, scale=0.3)
    np.testing.assert_array_equal(o_all[:, 1:2], o_ref)
    assert np.abs(o_all[:, 1:2] - o_alt).max() > 1e-3


def test_key_permutation_invariance():
    N, d = 23, 8
    q, k, v = rand(1, 2, N, d), rand(1, 2, N, d), rand(1, 2, N, d)
    perm = RNG.permutation(N)
    o1, l1 = oracle.attention(q, k, v, scale=0.4)
    o2, l2 = oracle.attention(q, k[:, :, perm], v[:, :, perm], scale=0.4)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-14)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-13)


def test_shift_invariance_large_offsets():
    # Adding u to every key adds scale*q.u to a row's scores: O is unchanged
    # and L moves by scale*q.u.  Offsets of ~1e3 overflow exp() unless the
    # maximum is subtracted first.
    N, d = 17, 4
    q, k, v = rand(1, 1, N, d), rand(1, 1, N, d), rand(1, 1, N, d)
    q = q * 40.0
    k = np.round(k * 64) / 64  # k + u stays exact in float32
    u = np.full(d, 25.0, dtype=np.float32)
    o1, l1 = oracle.attention(q, k, v, scale=0.5)
    o2, l2 = oracle.attention(q, k + u, v, scale=0.5)
    shift = 0.5 * (q[0, 0].astype(np.float64) @ u.astype(np.float64))
    assert np.isfinite(o2).all() and np.abs(shift).max() > 700
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-9)
    np.testing.assert_allclose(l2[0, 0], l1[0, 0] + shift, rtol=1e-14, atol=1e-9)


def test_causal_rows_equal_prefix_attention():
    N, d = 12, 4
    q, k, v = rand(1, 1, N, d), rand(1, 1, N, d), rand(1, 1, N, d)
    o, lse = oracle.attention(q, k, v, scale=0.8, causal=True)
    for i in range(N):
        oi, li = oracle.attention(q[:, :, i:i + 1], k[:, :, :i + 1], v[:, :, :i + 1], scale=0.8)
        np.testing.assert_array_equal(o[0, 0, i], oi[0, 0, 0])
        np.testing.assert_array_equal(lse[0, 0, i], li[0, 0, 0])


@pytest.mark.parametrize("causal", [False, True])
def test_row_evaluator_matches_full(causal):
    B, Hq, Hkv, N, d = 2, 4, 2, 33, 16
    q, k, v = rand(B, Hq, N, d), rand(B, Hkv, N, d), rand(B, Hkv, N, d)
    o, lse = oracle.attention(q, k, v, scale=0.25, causal=causal)
    rows = RNG.choice(B * Hq * N, size=40, replace=False)
    orow, lrow = oracle.attention_rows(q, k, v, 0.25, causal, rows)
    np.testing.assert_allclose(orow, o.reshape(-1, d)[rows], rtol=0, atol=1e-14)
    np.testing.assert_allclose(lrow, lse.reshape(-1)[rows], rtol=0, atol=1e-14)


def _bf16_bits(x):
    import torch
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _bits_to_f32(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32)


def test_paged_decode_equals_contiguous_and_is_placement_free():
    # Paging is memory management only: the same tokens scattered over two
    # different page placements give identical results, equal to attention
    # over the contiguous cache.
    S, Hq, Hkv, d, ps, P = 5, 8, 2, 16, 4, 40
    lens = np.array([1, 4, 5, 13, 0], dtype=np.int32)
    maxb = 4
    kc = [_bf16_bits(rand(Hkv, int(n), d)) for n in lens]
    vc = [_bf16_bits(rand(Hkv, int(n), d)) for n in lens]
    q = _bits_to_f32(_bf16_bits(rand(S, Hq, d)))
    results = []
    for seed in (1, 2):
        rng = np.random.default_rng(seed)
        perm = rng.permutation(P).astype(np.int32)
        kp = _bf16_bits(rand(P, Hkv, ps, d, rng=rng))  # unrelated filler everywhere
        vp = _bf16_bits(rand(P, Hkv, ps, d, rng=rng))
        bt = np.full((S, maxb), -1, dtype=np.int32)
        nxt = 0
        for s in range(S):
            n = -(-int(lens[s]) // ps)
            bt[s, :n] = perm[nxt:nxt + n]
            nxt += n
            for t in range(int(lens[s])):
                kp[bt[s, t // ps], :, t % ps] = kc[s][:, t]
                vp[bt[s, t // ps], :, t % ps] = vc[s][:, t]
        o, lse = oracle.decode_paged(q, kp, vp, bt, lens, scale=0.25)
        results.append((o, lse))
        for s in range(S):
            if lens[s] == 0:
                assert np.all(o[s] == 0) and np.all(np.isneginf(lse[s]))
                continue
            oc, lc = oracle.attention(q[s][None, :, None, :], _bits_to_f32(kc[s])[None],
                                      _bits_to_f32(vc[s])[None], scale=0.25)
            np.testing.assert_array_equal(o[s], oc[0, :, 0])
            np.testing.assert_array_equal(lse[s], lc[0, :, 0])
    np.testing.assert_array_equal(results[0][0], results[1][0])
    np.testing.assert_array_equal(results[0][1], results[1][1])


def test_decode_equals_causal_prefill_row():
    # Autoregressive check (Lab 01 "How to Test"): decoding token t against the
    # cache of tokens 0..t gives row t of the causal prefill.
    N, H, d, ps = 10, 2, 8, 4
    q = _bits_to_f32(_bf16_bits(rand(1, H, N, d)))
    kb, vb = _bf16_bits(rand(1, H, N, d)), _bf16_bits(rand(1, H, N, d))
    o, lse = oracle.attention(q, _bits_to_f32(kb), _bits_to_f32(vb), scale=0.35, causal=True)
    npages = -(-N // ps)
    kp = np.zeros((npages, H, ps, d), dtype=np.uint16)
    vp = np.zeros_like(kp)
    for t in range(N):
        kp[t // ps, :, t % ps] = kb[0, :, t]
        vp[t // ps, :, t % ps] = vb[0, :, t]
    bt = np.arange(npages, dtype=np.int32)[None]
    for t in range(N):
        od, ld = oracle.decode_paged(q[0, :, t][None], kp, vp, bt, np.array([t + 1], np.int32), scale=0.35)
        np.testing.assert_allclose(od[0], o[0, :, t], rtol=0, atol=1e-14)
        np.testing.assert_allclose(ld[0], lse[0, :, t], rtol=0, atol=1e-13)


def test_decode_rejects_bad_page_ids():
    kp = np.zeros((2, 1, 2, 1), dtype=np.uint16)
    with pytest.raises(ValueError):
        oracle.decode_paged(np.ones((1, 1, 1), np.float32), kp, kp,
                            np.array([[0, 5]], np.int32), np.array([3], np.int32), scale=1.0)


# ------------------------------------------------------- FP8 (e4m3) KV cache


def _e4m3_table():
    """All 256 E4M3 bytes decoded by torch's float8_e4m3fn conversion (an
    implementation independent of the oracle), as float64."""
    import torch
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    return codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_e4m3_decoding_matches_format():
    # The format's fixed points: 1.0 = 0.0111.000, the largest finite value 448
    # = 0.1111.110, the smallest normal 2^-6, the smallest subnormal 2^-9,
    # NaN at S.1111.111, sign-magnitude negatives; then all 256 codes against
    # torch's converter.
    assert oracle.e4m3_to_double(0x38) == 1.0
    assert oracle.e4m3_to_double(0x7E) == 448.0
    assert oracle.e4m3_to_double(0x08) == 2.0 ** -6
    assert oracle.e4m3_to_double(0x01) == 2.0 ** -9
    assert oracle.e4m3_to_double(0x07) == 7 * 2.0 ** -9
    assert oracle.e4m3_to_double(0x3C) == 1.5
    assert oracle.e4m3_to_double(0xC0) == -2.0
    assert math.isnan(oracle.e4m3_to_double(0x7F)) and math.isnan(oracle.e4m3_to_double(0xFF))
    assert math.copysign(1.0, oracle.e4m3_to_double(0x80)) == -1.0
    ref = _e4m3_table()
    got = np.array([oracle.e4m3_to_double(b) for b in range(256)])
    finite = ~np.isnan(ref)
    np.testing.assert_array_equal(np.isnan(got), ~finite)
    np.testing.assert_array_equal(got[finite], ref[finite])


def _q8_cache(rng, P, Hkv, ps, d, scale_exps, fmt):
    """Random finite 8-bit codes (E4M3 NaN codes excluded) and power-of-two scales."""
    kb = rng.integers(0, 256, size=(P, Hkv, ps, d)).astype(np.uint8)
    vb = rng.integers(0, 256, size=(P, Hkv, ps, d)).astype(np.uint8)
    if fmt == "e4m3":
        for a in (kb, vb):
            a[(a & 0x7F) == 0x7F] = 0x3A
    ks = (2.0 ** rng.choice(scale_exps, size=(P, Hkv))).astype(np.float32)
    vs = (2.0 ** rng.choice(scale_exps, size=(P, Hkv))).astype(np.float32)
    return kb, vb, ks, vs


def _q8_values(codes, fmt):
    """Decoded codes, by torch's e4m3 converter or numpy's int8 view."""
    if fmt == "e4m3":
        return _e4m3_table()[codes]
    return codes.view(np.int8).astype(np.float64)


@pytest.mark.parametrize("fmt", ["e4m3", "int8"])
def test_q8_decode_equals_decode_of_dequantised_cache(fmt):
    # With per-(page, head) scales, each cached element is scale * code.
    # Dequantise in the test (torch's e4m3 table or numpy's int8 view); with
    # power-of-two scales every value is exactly representable in bf16 (at
    # most 8 significant bits), so the pinned bf16 paged decode sees the same
    # numbers and must agree exactly.
    rng = np.random.default_rng(77)
    S, Hq, Hkv, d, ps, P, maxb = 4, 8, 2, 16, 4, 24, 5
    exps = [-6, -5, -4, -3] if fmt == "e4m3" else [-9, -8, -7]
    kb, vb, ks, vs = _q8_cache(rng, P, Hkv, ps, d, exps, fmt)
    lens = np.array([1, 7, 20, 0], dtype=np.int32)
    bt = np.full((S, maxb), -1, dtype=np.int32)
    perm = rng.permutation(P).astype(np.int32)
    nxt = 0
    for s in range(S):
        n = -(-int(lens[s]) // ps)
        bt[s, :n] = perm[nxt:nxt + n]
        nxt += n
    q = _bits_to_f32(_bf16_bits(rand(S, Hq, d, rng=rng)))
    kd = _q8_values(kb, fmt) * ks[:, :, None, None].astype(np.float64)
    vd = _q8_values(vb, fmt) * vs[:, :, None, None].astype(np.float64)
    kbits, vbits = _bf16_bits(kd.astype(np.float32)), _bf16_bits(vd.astype(np.float32))
    np.testing.assert_array_equal(_bits_to_f32(kbits).astype(np.float64), kd)
    np.testing.assert_array_equal(_bits_to_f32(vbits).astype(np.float64), vd)
    o8, l8 = oracle.decode_paged_q8(q, kb, vb, ks, vs, bt, lens, scale=0.3, fmt=fmt)
    ob, lb = oracle.decode_paged(q, kbits, vbits, bt, lens, scale=0.3)
    np.testing.assert_array_equal(o8, ob)
    np.testing.assert_array_equal(l8, lb)
    # and directly against contiguous attention over the dequantised tokens
    for s in range(S):
        if lens[s] == 0:
            continue
        n = int(lens[s])
        kc = np.stack([kd[bt[s, t // ps], :, t % ps] for t in range(n)], axis=1)
        vc = np.stack([vd[bt[s, t // ps], :, t % ps] for t in range(n)], axis=1)
        oc, lc = oracle.attention(q[s][None, :, None, :], kc[None], vc[None], scale=0.3)
        np.testing.assert_allclose(o8[s], oc[0, :, 0], rtol=0, atol=1e-12)
        np.testing.assert_allclose(l8[s], lc[0, :, 0], rtol=0, atol=1e-12)


@pytest.mark.parametrize("fmt", ["e4m3", "int8"])
def test_q8_scale_linearity(fmt):
    # V's scale multiplies the output and leaves L alone; K's scale multiplies
    # every score, i.e. acts like the softmax scale.
    rng = np.random.default_rng(78)
    S, Hq, Hkv, d, ps, P, maxb = 2, 4, 2, 8, 4, 6, 3
    kb, vb, _, _ = _q8_cache(rng, P, Hkv, ps, d, [0], fmt)
    one = np.ones((P, Hkv), np.float32)
    bt = np.array([[0, 1, 2], [3, 4, 5]], dtype=np.int32)
    lens = np.array([9, 12], dtype=np.int32)
    q = rand(S, Hq, d, rng=rng) * (0.05 if fmt == "e4m3" else 0.002)
    o1, l1 = oracle.decode_paged_q8(q, kb, vb, one, one, bt, lens, scale=0.5, fmt=fmt)
    o2, l2 = oracle.decode_paged_q8(q, kb, vb, one, 3.0 * one, bt, lens, scale=0.5, fmt=fmt)
    np.testing.assert_allclose(o2, 3.0 * o1, rtol=1e-13, atol=1e-13)
    np.testing.assert_array_equal(l2, l1)
    o3, l3 = oracle.decode_paged_q8(q, kb, vb, 0.25 * one, one, bt, lens, scale=0.5, fmt=fmt)
    o4, l4 = oracle.decode_paged_q8(q, kb, vb, one, one, bt, lens, scale=0.125, fmt=fmt)
    np.testing.assert_allclose(o3, o4, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l3, l4, rtol=0, atol=1e-12)


def test_q8_decode_rejects_bad_page_ids():
    kp = np.zeros((2, 1, 2, 1), dtype=np.uint8)
    sc = np.ones((2, 1), np.float32)
    with pytest.raises(ValueError):
        oracle.decode_paged_q8(np.ones((1, 1, 1), np.float32), kp, kp, sc, sc,
                               np.array([[0, 5]], np.int32), np.array([3], np.int32), scale=1.0)


# --------------------------------------------------------- chunked prefill


def _paged_case(lens, qlens, Hq, Hkv, d, ps=4, seed=0):
    """A page pool holding each sequence's tokens in shuffled pages, and the
    contiguous copies (bf16 values) for the checks."""
    rng = np.random.default_rng(seed)
    S = len(lens)
    maxb = max(1, max(-(-n // ps) for n in lens))
    P = sum(-(-n // ps) for n in lens) + 3
    kp = _bf16_bits(rand(P, Hkv, ps, d, rng=rng))
    vp = _bf16_bits(rand(P, Hkv, ps, d, rng=rng))
    perm = rng.permutation(P).astype(np.int32)
    bt = np.full((S, maxb), -1, dtype=np.int32)
    nxt = 0
    kc, vc = [], []
    for s_, n in enumerate(lens):
        k = -(-n // ps)
        bt[s_, :k] = perm[nxt:nxt + k]
        nxt += k
        kc.append(np.stack([_bits_to_f32(kp[bt[s_, t // ps], :, t % ps]) for t in range(n)], axis=1)
                  if n else np.zeros((Hkv, 0, d), np.float32))
        vc.append(np.stack([_bits_to_f32(vp[bt[s_, t // ps], :, t % ps]) for t in range(n)], axis=1)
                  if n else np.zeros((Hkv, 0, d), np.float32))
    cu = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    q = _bits_to_f32(_bf16_bits(rand(int(cu[-1]), Hq, d, rng=rng)))
    return q, kp, vp, bt, np.array(lens, np.int32), cu, kc, vc


def test_prefill_paged_equals_causal_rows_of_full_prefill():
    # The chunk's queries placed at rows ctx..len-1 of a full causal prefill
    # over the contiguous sequence give those rows (rows before ctx arbitrary).
    lens, qlens = [9, 13, 5, 4], [3, 13, 1, 0]
    Hq, Hkv, d = 4, 2, 8
    q, kp, vp, bt, sl, cu, kc, vc = _paged_case(lens, qlens, Hq, Hkv, d, seed=51)
    o, lse = oracle.prefill_paged(q, kp, vp, bt, sl, cu, scale=0.3)
    rng = np.random.default_rng(52)
    for s_, (n, ql) in enumerate(zip(lens, qlens)):
        if ql == 0:
            continue
        ctx = n - ql
        qf = rand(1, Hq, n, d, rng=rng)
        qf[0, :, ctx:] = q[cu[s_]:cu[s_ + 1]].transpose(1, 0, 2)
        of, lf = oracle.attention(qf, kc[s_][None], vc[s_][None], scale=0.3, causal=True)
        np.testing.assert_allclose(o[cu[s_]:cu[s_ + 1]], of[0, :, ctx:].transpose(1, 0, 2),
                                   rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse[cu[s_]:cu[s_ + 1]], lf[0, :, ctx:].T, rtol=0, atol=1e-13)


def test_prefill_paged_single_query_is_decode():
    lens, qlens = [7, 1, 12], [1, 1, 1]
    q, kp, vp, bt, sl, cu, _, _ = _paged_case(lens, qlens, 4, 1, 8, seed=53)
    o, lse = oracle.prefill_paged(q, kp, vp, bt, sl, cu, scale=0.5)
    od, ld = oracle.decode_paged(q, kp, vp, bt, sl, scale=0.5)
    np.testing.assert_allclose(o, od, rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse, ld, rtol=0, atol=1e-14)


def test_prefill_paged_chunking_invariance():
    # Processing a prompt chunk in two pieces (the first piece with the
    # shorter length) gives the same rows as processing it at once.
    n, ql, split = 14, 9, 4
    q, kp, vp, bt, sl, cu, _, _ = _paged_case([n], [ql], 2, 2, 8, seed=54)
    o, lse = oracle.prefill_paged(q, kp, vp, bt, sl, cu, scale=0.4)
    o1, l1 = oracle.prefill_paged(q[:split], kp, vp, bt, np.array([n - ql + split], np.int32),
                                  np.array([0, split], np.int32), scale=0.4)
    o2, l2 = oracle.prefill_paged(q[split:], kp, vp, bt, np.array([n], np.int32),
                                  np.array([0, ql - split], np.int32), scale=0.4)
    np.testing.assert_array_equal(np.concatenate([o1, o2]), o)
    np.testing.assert_array_equal(np.concatenate([l1, l2]), lse)


def test_prefill_paged_rejects_chunk_longer_than_sequence():
    q, kp, vp, bt, sl, cu, _, _ = _paged_case([5], [5], 1, 1, 4, seed=55)
    with pytest.raises(ValueError):
        oracle.prefill_paged(q, kp, vp, bt, np.array([4], np.int32), cu, scale=1.0)


# ------------------------------------------------------------------ backward


def _grid_values(rng, shape, denom=1024):
    """Values k/denom with |k| < denom/2: exact in float32, and so is x +- 2h for
    h = 2^-12, which the finite-difference stencil below needs."""
    return (rng.integers(-denom // 2, denom // 2, shape) / denom).astype(np.float32)


def _fd_grads(q, k, v, do, scale, causal=False, window=0, alibi_slopes=None):
    """Gradients of sum(do * O) by the 4-point central stencil (error O(h^4)),
    from forward evaluations only."""
    h = 2.0 ** -12
    dod = do.astype(np.float64)

    def f(a):
        o, _ = oracle.attention(a[0], a[1], a[2], scale=scale, causal=causal, window=window,
                                alibi_slopes=alibi_slopes)
        return float((o * dod).sum())

    out = []
    for which in range(3):
        base = [q, k, v]
        g = np.zeros(base[which].shape)
        for idx in np.ndindex(base[which].shape):
            def ev(delta):
                a = [x.copy() for x in base]
                a[which][idx] += np.float32(delta)
                return f(a)
            g[idx] = (8 * (ev(h) - ev(-h)) - (ev(2 * h) - ev(-2 * h))) / (12 * h)
        out.append(g)
    return out


@pytest.mark.parametrize("causal,window,alibi,Hq,Hkv", [
    (False, 0, False, 1, 1), (True, 0, False, 2, 1), (True, 3, True, 2, 2), (False, 0, True, 4, 2)])
def test_bwd_matches_finite_differences(causal, window, alibi, Hq, Hkv):
    # The backward is the derivative of the forward: compare with a numerical
    # derivative of the (separately pinned) forward oracle.
    rng = np.random.default_rng(31 + Hq + window)
    B, N, d = 1, 6, 3
    q, k, v = (_grid_values(rng, (B, Hq, N, d)), _grid_values(rng, (B, Hkv, N, d)),
               _grid_values(rng, (B, Hkv, N, d)))
    do = _grid_values(rng, (B, Hq, N, d))
    slopes = [0.5 * (h + 1) for h in range(Hq)] if alibi else None
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, scale=0.7, causal=causal, window=window,
                                      alibi_slopes=slopes)
    fq, fk, fv = _fd_grads(q, k, v, do, 0.7, causal, window, slopes)
    for got, ref in ((dq, fq), (dk, fk), (dv, fv)):
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-10)


def test_bwd_two_keys_closed_form():
    # One query, two keys: P = (sig, 1 - sig) with sig the logistic of s0 - s1,
    # dV_j = P_j dO, dS_0 = -dS_1 = sig (1 - sig) dO.(v0 - v1),
    # dQ = scale dS_0 (k0 - k1), dK_0 = -dK_1 = scale dS_0 q.
    q = np.array([[[[0.5, -0.25]]]], np.float32)
    k = np.array([[[[1.0, 0.5], [-0.5, 0.25]]]], np.float32)
    v = np.array([[[[2.0, 0.0], [0.0, -1.0]]]], np.float32)
    # a second query row that sees both keys too (non-causal), with zero dO
    q2 = np.concatenate([q, np.zeros_like(q)], axis=2)
    do = np.array([[[[1.0, 3.0], [0.0, 0.0]]]], np.float32)
    scale = 0.8
    dq, dk, dv = oracle.attention_bwd(q2, k, v, do, scale=scale)
    s0 = scale * float(q[0, 0, 0] @ k[0, 0, 0]); s1 = scale * float(q[0, 0, 0] @ k[0, 0, 1])
    sig = 1.0 / (1.0 + math.exp(-(s0 - s1)))
    dO = do[0, 0, 0].astype(np.float64)
    ds0 = sig * (1 - sig) * float(dO @ (v[0, 0, 0] - v[0, 0, 1]))
    np.testing.assert_allclose(dv[0, 0, 0], sig * dO, atol=1e-15)
    np.testing.assert_allclose(dv[0, 0, 1], (1 - sig) * dO, atol=1e-15)
    np.testing.assert_allclose(dq[0, 0, 0], scale * ds0 * (k[0, 0, 0] - k[0, 0, 1]), atol=1e-15)
    np.testing.assert_allclose(dk[0, 0, 0], scale * ds0 * q[0, 0, 0], atol=1e-15)
    np.testing.assert_allclose(dk[0, 0, 1], -scale * ds0 * q[0, 0, 0], atol=1e-15)
    assert np.all(dq[0, 0, 1] == 0)


@pytest.mark.parametrize("causal,window", [(False, 0), (True, 0), (True, 5)])
def test_bwd_invariants(causal, window):
    # Adding one vector to every key shifts each score row by a constant, so the
    # dK of a head sum to zero; every P row sums to one, so the dV sum to the
    # dO sum; with all values equal, O is constant and dQ = dK = 0.
    rng = np.random.default_rng(41)
    B, Hq, Hkv, N, d = 2, 4, 2, 19, 8
    q, k, v = rand(B, Hq, N, d, rng=rng), rand(B, Hkv, N, d, rng=rng), rand(B, Hkv, N, d, rng=rng)
    do = rand(B, Hq, N, d, rng=rng)
    slopes = [0.1 * (h + 1) for h in range(Hq)]
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, scale=0.3, causal=causal, window=window,
                                      alibi_slopes=slopes)
    np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-12)
    G = Hq // Hkv
    dosum = do.astype(np.float64).reshape(B, Hkv, G, N, d).sum(axis=(2, 3))
    np.testing.assert_allclose(dv.sum(axis=2), dosum, atol=1e-11)
    vc = np.broadcast_to(rand(B, Hkv, 1, d, rng=rng), v.shape).copy()
    dq2, dk2, _ = oracle.attention_bwd(q, k, vc, do, scale=0.3, causal=causal, window=window)
    assert np.abs(dq2).max() < 1e-13 and np.abs(dk2).max() < 1e-13


def test_bwd_gqa_equals_mha_with_summed_heads():
    rng = np.random.default_rng(42)
    B, Hq, Hkv, N, d = 1, 6, 2, 11, 4
    q, k, v = rand(B, Hq, N, d, rng=rng), rand(B, Hkv, N, d, rng=rng), rand(B, Hkv, N, d, rng=rng)
    do = rand(B, Hq, N, d, rng=rng)
    G = Hq // Hkv
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, scale=0.4, causal=True)
    kr, vr = np.repeat(k, G, axis=1), np.repeat(v, G, axis=1)
    dq2, dk2, dv2 = oracle.attention_bwd(q, kr, vr, do, scale=0.4, causal=True)
    np.testing.assert_allclose(dq, dq2, atol=1e-14)
    np.testing.assert_allclose(dk, dk2.reshape(B, Hkv, G, N, d).sum(axis=2), atol=1e-13)
    np.testing.assert_allclose(dv, dv2.reshape(B, Hkv, G, N, d).sum(axis=2), atol=1e-13)


@pytest.mark.parametrize("causal,window,alibi", [(False, 0, False), (True, 0, False), (True, 7, True)])
def test_bwd_sampled_evaluators_match_full(causal, window, alibi):
    rng = np.random.default_rng(43)
    B, Hq, Hkv, N, d = 2, 4, 2, 37, 16
    q, k, v = rand(B, Hq, N, d, rng=rng), rand(B, Hkv, N, d, rng=rng), rand(B, Hkv, N, d, rng=rng)
    do = rand(B, Hq, N, d, rng=rng)
    slopes = [0.05 * (h + 1) for h in range(Hq)] if alibi else None
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, scale=0.25, causal=causal, window=window,
                                      alibi_slopes=slopes)
    rows = np.array([0, 1, 36, 37, 80, B * Hq * N - 1])
    got = oracle.attention_bwd_dq_rows(q, k, v, do, 0.25, causal, rows, window=window,
                                       alibi_slopes=slopes)
    np.testing.assert_allclose(got, dq.reshape(-1, d)[rows], rtol=0, atol=1e-13)
    keys = np.array([0, 5, 36, 37, 74, B * Hkv * N - 1])
    gk, gv = oracle.attention_bwd_dkv_rows(q, k, v, do, 0.25, causal, keys, window=window,
                                           alibi_slopes=slopes)
    np.testing.assert_allclose(gk, dk.reshape(-1, d)[keys], rtol=0, atol=1e-12)
    np.testing.assert_allclose(gv, dv.reshape(-1, d)[keys], rtol=0, atol=1e-12)


# ------------------------------------------------------------- mutations

MUTANTS = {
    "no_max_shift_sign": ("s[j] = exp(s[j] - m)", "s[j] = exp(m - s[j])"),
    "drop_normalisation": ("double p = s[j] / l;", "double p = s[j];"),
    "lse_without_max": ("*lse = m + log(l);", "*lse = log(l);"),
    "causal_off_by_one": ("*hi = causal ? ((i + 1 < Nk) ? i + 1 : Nk) : Nk;",
                          "*hi = causal ? ((i < Nk) ? i + (i == 0) : Nk) : Nk;"),
    "window_off_by_one": ("i - window + 1 > 0) ? i - window + 1 : 0;", "i - window > 0) ? i - window : 0;"),
    "alibi_sign": ("S[(size_t)i * Nk + j] += slopes[h] * (double)(j - i);",
                   "S[(size_t)i * Nk + j] += slopes[h] * (double)(i - j);"),
    "wrong_gqa_group": ("int g = h / G;\n            const float *qh", "int g = h % Hkv;\n            const float *qh"),
    "dropped_term": ("for (c = 0; c < d; ++c) acc += Qd", "for (c = 1; c < d; ++c) acc += Qd"),
    "log_base_two": ("*lse = m + log(l);", "*lse = m + log2(l);"),
    "scale_dropped": ("S[(size_t)i * Nk + j] = scale * acc;", "S[(size_t)i * Nk + j] = acc;"),
}


Q8_MUTANTS = {
    "e4m3_bias": ("else v = ldexp(1.0 + (double)m / 8.0, e - 7);",
                  "else v = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    "e4m3_subnormal_exponent": ("if (e == 0) v = ldexp((double)m / 8.0, -6);",
                                "if (e == 0) v = ldexp((double)m / 8.0, -7);"),
    "e4m3_mantissa_width": ("else v = ldexp(1.0 + (double)m / 8.0, e - 7);",
                            "else v = ldexp(1.0 + (double)m / 16.0, e - 7);"),
    "q8_scales_swapped": ("double ks = (double)k_scales[(size_t)p * Hkv + g];",
                          "double ks = (double)v_scales[(size_t)p * Hkv + g];"),
    "q8_scale_index": ("double vs = (double)v_scales[(size_t)p * Hkv + g];",
                       "double vs = (double)v_scales[(size_t)g * Hkv + p % Hkv];"),
    "int8_unsigned": ("fmt == 0 ? e4m3_to_double(b) : (double)(int8_t)b;",
                      "fmt == 0 ? e4m3_to_double(b) : (double)b;"),
}


def _run_mutant(src_old, src_new, tmp_path, checks):
    src = open(os.path.join(ROOT, "oracle", "attn_oracle.c")).read()
    assert src_old in src
    mutated = src.replace(src_old, src_new, 1)
    cpath = tmp_path / "mut.c"
    cpath.write_text(mutated)
    lib = tmp_path / "libmut.so"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", str(lib), str(cpath), "-lm"])
    saved = oracle._lib
    real_build = oracle.build
    try:
        oracle._lib = None
        oracle.build = lambda force=False: str(lib)
        failures = 0
        for chk in checks:
            try:
                chk()
            except (AssertionError, ValueError, FloatingPointError):
                failures += 1
        return failures
    finally:
        oracle.build = real_build
        oracle._lib = saved


PAGED_PREFILL_MUTANTS = {
    "chunk_visible_off_by_one": ("int nvis = ctx + t + 1, j;", "int nvis = ctx + t, j;"),
    "chunk_ctx_ignored": ("int ctx = len - ql, t, c, hh;", "int ctx = 0, t, c, hh;"),
    "chunk_wrong_query_row": ("const float *qt = q + ((size_t)(q0 + t) * Hq + h) * (size_t)d;",
                              "const float *qt = q + ((size_t)(t) * Hq + h) * (size_t)d;"),
}


@pytest.mark.parametrize("name", sorted(PAGED_PREFILL_MUTANTS))
def test_prefill_paged_pins_catch_planted_mistakes(name, tmp_path):
    old, new = PAGED_PREFILL_MUTANTS[name]
    checks = [test_prefill_paged_equals_causal_rows_of_full_prefill,
              test_prefill_paged_single_query_is_decode, test_prefill_paged_chunking_invariance]
    assert _run_mutant(old, new, tmp_path, checks) > 0, "mutant %s survived every pin" % name


BWD_MUTANTS = {
    "bwd_drop_D": ("for (j = lo; j < hi; ++j) dSi[j] = Pi[j] * (dSi[j] - D);",
                   "for (j = lo; j < hi; ++j) dSi[j] = Pi[j] * dSi[j];"),
    "bwd_dq_unscaled": ("dqi[c] = scale * acc;", "dqi[c] = acc;"),
    "bwd_dk_uses_P": ("ak += dS[(size_t)r * N + i] * Qd[(size_t)r * d + c];",
                      "ak += P[(size_t)r * N + i] * Qd[(size_t)r * d + c];"),
    "bwd_dv_transposed": ("av += P[(size_t)r * N + i] * dOd[(size_t)r * d + c];",
                          "av += P[(size_t)i * N + r] * dOd[(size_t)r * d + c];"),
    "bwd_dk_not_summed_over_group": ("dkj[c] += scale * ak;", "dkj[c] = scale * ak;"),
    "bwd_rows_sign": ("acc += s[j - lo] * (dp[j - lo] - D) * Kd[(size_t)j * d + c];",
                      "acc += s[j - lo] * (D - dp[j - lo]) * Kd[(size_t)j * d + c];"),
    "bwd_keys_missing_alibi": ("p = exp(scale * sc + (slopes ? slopes[h] : 0.0) * (double)(j - i) - L[(size_t)hh * N + i]);",
                               "p = exp(scale * sc - L[(size_t)hh * N + i]);"),
}


@pytest.mark.parametrize("name", sorted(BWD_MUTANTS))
def test_bwd_pins_catch_planted_mistakes(name, tmp_path):
    old, new = BWD_MUTANTS[name]
    checks = [lambda: test_bwd_matches_finite_differences(True, 3, True, 2, 2),
              lambda: test_bwd_matches_finite_differences(False, 0, False, 1, 1),
              lambda: test_bwd_matches_finite_differences(False, 0, True, 4, 2),
              test_bwd_two_keys_closed_form, test_bwd_gqa_equals_mha_with_summed_heads,
              lambda: test_bwd_sampled_evaluators_match_full(True, 7, True),
              lambda: test_bwd_invariants(True, 0)]
    assert _run_mutant(old, new, tmp_path, checks) > 0, "mutant %s survived every pin" % name


@pytest.mark.parametrize("name", sorted(Q8_MUTANTS))
def test_q8_pins_catch_planted_mistakes(name, tmp_path):
    old, new = Q8_MUTANTS[name]
    checks = [test_e4m3_decoding_matches_format]
    for fmt in ("e4m3", "int8"):
        checks += [lambda f=fmt: test_q8_decode_equals_decode_of_dequantised_cache(f),
                   lambda f=fmt: test_q8_scale_linearity(f)]
    assert _run_mutant(old, new, tmp_path, checks) > 0, "mutant %s survived every pin" % name


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistakes(name, tmp_path):
    """Each mutant of the oracle's C source fails at least one closed-form pin."""
    src = open(os.path.join(ROOT, "oracle", "attn_oracle.c")).read()
    old, new = MUTANTS[name]
    assert old in src, name
    mutated = src.replace(old, new, 1)
    cpath = tmp_path / "mut.c"
    cpath.write_text(mutated)
    lib = tmp_path / "libmut.so"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", str(lib), str(cpath), "-lm"])
    saved = oracle._lib
    try:
        oracle._lib = None
        real_build = oracle.build
        oracle.build = lambda force=False: str(lib)
        failures = 0
        checks = [test_window_of_one_returns_own_value,
                  lambda: test_alibi_is_one_extra_dimension(True),
                  lambda: test_decimal_brute_force_window_alibi(2, True),
                  test_window_rows_equal_attention_over_the_window,
                  test_single_key_returns_its_value, test_identical_keys_average_the_values,
                  lambda: test_weights_sum_to_one(True), test_causal_row_zero_sees_only_key_zero,
                  test_two_keys_logistic_weights, test_gqa_equals_mha_with_repeated_heads,
                  lambda: test_decimal_brute_force(5, 4, 2, 2, True),
                  lambda: test_decimal_brute_force(8, 3, 4, 2, False),
                  test_causal_rows_equal_prefix_attention]
        for golden in _golden()["prefill"]:
            checks.append(lambda g=golden: test_golden_prefill(g))
        for chk in checks:
            try:
                chk()
            except (AssertionError, ValueError, FloatingPointError):
                failures += 1
        assert failures > 0, "mutant %s survived every pin" % name
    finally:
        oracle.build = real_build
        oracle._lib = saved


def test_wrappers_refuse_tensors_that_disagree():
    # The C code trusts the sizes it is given, so the wrappers compare every
    # tensor with q's shape before calling it (a mismatch would read past an
    # array instead of failing).
    z = np.zeros
    q = z((1, 2, 4, 8), np.float32)
    with pytest.raises(ValueError):
        oracle.attention(q, z((2, 1, 4, 8)), z((2, 1, 4, 8)), scale=1.0)   # other B
    with pytest.raises(ValueError):
        oracle.attention(q, z((1, 1, 4, 16)), z((1, 1, 4, 16)), scale=1.0)  # other d
    with pytest.raises(ValueError):
        oracle.attention(q, z((1, 1, 4, 8)), z((1, 1, 3, 8)), scale=1.0)   # v unlike k
    with pytest.raises(ValueError):
        oracle.attention_rows(q, z((1, 1, 4, 8)), z((1, 1, 5, 8)), 1.0, False, [0])
    for fn, extra in ((oracle.attention_bwd, ()), (oracle.attention_bwd_dq_rows, (False, [0])),
                      (oracle.attention_bwd_dkv_rows, (False, [0]))):
        with pytest.raises(ValueError):
            fn(q, z((1, 1, 4, 8)), z((1, 1, 4, 8)), z((1, 2, 3, 8)), 1.0, *extra)  # dO unlike q
        with pytest.raises(ValueError):
            fn(q, z((1, 1, 5, 8)), z((1, 1, 5, 8)), q, 1.0, *extra)  # keys unlike queries
    qd = z((3, 2, 8), np.float32)
    pages = z((4, 1, 16, 8), np.uint16)
    bt, sl = z((3, 2), np.int32), z(3, np.int32)
    with pytest.raises(ValueError):
        oracle.decode_paged(qd, pages, pages, bt[:2], sl, scale=1.0)
    with pytest.raises(ValueError):
        oracle.decode_paged(qd, pages, pages, bt, sl[:2], scale=1.0)
    sc = np.ones((4, 1), np.float32)
    with pytest.raises(ValueError):
        oracle.decode_paged_q8(qd, pages.astype(np.uint8), pages.astype(np.uint8), sc, sc,
                               bt[:1], sl, scale=1.0)
    with pytest.raises(ValueError):
        oracle.prefill_paged(qd, pages, pages, bt[:2], sl, z(4, np.int32) + [0, 1, 2, 3],
                             scale=1.0)
