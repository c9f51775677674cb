"""fp64 CPU oracle for exact attention -- test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
arm of ``bench.py`` may import this package.  It never imports the CUDA
package and shares no code with it; the two meet only through the seeded input
generators, which hold none of the method's arithmetic.

The arithmetic lives in ``attn_oracle.c`` (plain C, fp64, OpenMP); this module
compiles it with gcc on first use and marshals numpy arrays to it.  It covers
the forward (full and sampled rows), the paged decode over 16-bit and 8-bit
caches, and the backward (full, sampled dQ rows, sampled dK/dV keys).  The
definition it evaluates is standard attention (Phase 08 page, Lab 01 step 1;
screna.ai FlashAttention answer): S = scale * Q K^T over the visible keys,
P = softmax(S) row-wise, O = P V, L = m + ln(sum exp(s - m)).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile attn_oracle.c into liboracle.so (gcc, -O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or (
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        f32p = ctypes.POINTER(ctypes.c_float)
        f64p = ctypes.POINTER(ctypes.c_double)
        i32p = ctypes.POINTER(ctypes.c_int32)
        i64p = ctypes.POINTER(ctypes.c_int64)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        ci, cd = ctypes.c_int, ctypes.c_double
        lib.oracle_attn.argtypes = [f32p, f32p, f32p, f64p, f64p,
                                    ci, ci, ci, ci, ci, ci, cd, ci, ci, f64p, ci]
        lib.oracle_attn.restype = ci
        lib.oracle_attn_rows.argtypes = [f32p, f32p, f32p, f64p, f64p,
                                         ci, ci, ci, ci, ci, ci, cd, ci, ci, f64p,
                                         i64p, ci, ci]
        lib.oracle_attn_rows.restype = ci
        lib.oracle_decode_paged.argtypes = [f32p, u16p, u16p, i32p, i32p, f64p, f64p,
                                            ci, ci, ci, ci, ci, ci, ci, cd,
                                            i32p, ci, ci]
        lib.oracle_decode_paged.restype = ci
        u8p = ctypes.POINTER(ctypes.c_uint8)
        lib.oracle_decode_paged_q8.argtypes = [f32p, u8p, u8p, f32p, f32p, i32p, i32p, f64p,
                                               f64p, ci, ci, ci, ci, ci, ci, ci, cd, ci,
                                               i32p, ci, ci]
        lib.oracle_decode_paged_q8.restype = ci
        lib.oracle_e4m3_to_double.argtypes = [ci]
        lib.oracle_e4m3_to_double.restype = cd
        lib.oracle_prefill_paged.argtypes = [f32p, u16p, u16p, i32p, i32p, i32p, f64p, f64p,
                                             ci, ci, ci, ci, ci, ci, ci, cd, ci]
        lib.oracle_prefill_paged.restype = ci
        lib.oracle_attn_bwd.argtypes = [f32p, f32p, f32p, f32p, f64p, f64p, f64p,
                                        ci, ci, ci, ci, ci, cd, ci, ci, f64p, ci]
        lib.oracle_attn_bwd.restype = ci
        lib.oracle_attn_bwd_dq_rows.argtypes = [f32p, f32p, f32p, f32p, f64p, ci, ci, ci, ci, ci,
                                                cd, ci, ci, f64p, i64p, ci, ci]
        lib.oracle_attn_bwd_dq_rows.restype = ci
        lib.oracle_attn_bwd_dkv_rows.argtypes = [f32p, f32p, f32p, f32p, f64p, f64p, ci, ci, ci,
                                                 ci, ci, cd, ci, ci, f64p, i64p, ci, ci]
        lib.oracle_attn_bwd_dkv_rows.restype = ci
        lib.oracle_max_threads.argtypes = []
        lib.oracle_max_threads.restype = ci
        _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def _slopes(slopes, Hq):
    if slopes is None:
        return None
    a = np.ascontiguousarray(np.asarray(slopes, dtype=np.float64).reshape(-1))
    if a.size != Hq:
        raise ValueError("need one ALiBi slope per query head")
    return a


def _sp(a):
    return None if a is None else _ptr(a, ctypes.c_double)


def _qkv_dims(q, k, v, *more):
    """(B, Hq, Hkv, Nq, Nk, d) of q [B,Hq,Nq,d] and k, v [B,Hkv,Nk,d]; the C code
    trusts these sizes, so tensors that disagree are refused here.  ``more``
    are tensors that must have q's shape (dO)."""
    if q.ndim != 4 or k.ndim != 4 or v.ndim != 4:
        raise ValueError("q, k, v must be 4-D")
    B, Hq, Nq, d = q.shape
    if k.shape[0] != B or k.shape[3] != d or v.shape != k.shape:
        raise ValueError("k and v must be [B, Hkv, Nk, d] with q's B and d")
    for t in more:
        if t.shape != q.shape:
            raise ValueError("shape mismatch")
    return B, Hq, k.shape[1], Nq, k.shape[2], d


def _table_dims(S, bt, sl):
    if bt.ndim != 2 or sl.ndim != 1 or bt.shape[0] != S or sl.size != S:
        raise ValueError("block_table must be [S, max_blocks] and seq_lens [S]")


def attention(q, k, v, scale: float, causal: bool = False, nthreads: int | None = None,
              window: int = 0, alibi_slopes=None):
    """Standard attention in fp64.  q [B,Hq,Nq,d], k/v [B,Hkv,Nk,d] (float32 values).

    Returns (O [B,Hq,Nq,d] float64, L [B,Hq,Nq] float64).  Causal: key j is
    visible to query i iff j <= i.  window W > 0 keeps keys with i - j < W;
    alibi_slopes (one per query head) add slope_h * (j - i) to the scores.
    """
    q, k, v = _f32(q), _f32(k), _f32(v)
    B, Hq, Hkv, Nq, Nk, d = _qkv_dims(q, k, v)
    o = np.zeros((B, Hq, Nq, d), dtype=np.float64)
    lse = np.zeros((B, Hq, Nq), dtype=np.float64)
    sl = _slopes(alibi_slopes, Hq)
    rc = _load().oracle_attn(_ptr(q, ctypes.c_float), _ptr(k, ctypes.c_float),
                             _ptr(v, ctypes.c_float), _ptr(o, ctypes.c_double),
                             _ptr(lse, ctypes.c_double), B, Hq, Hkv, Nq, Nk, d,
                             float(scale), int(bool(causal)), int(window), _sp(sl),
                             int(nthreads or max_threads()))
    if rc != 0:
        raise ValueError("oracle_attn failed with code %d" % rc)
    return o, lse


def attention_rows(q, k, v, scale: float, causal: bool, rows, nthreads: int | None = None,
                   window: int = 0, alibi_slopes=None):
    """The same definition for selected rows; rows[r] = (b*Hq + h)*Nq + i."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    B, Hq, Hkv, Nq, Nk, d = _qkv_dims(q, k, v)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    o = np.zeros((rows.size, d), dtype=np.float64)
    lse = np.zeros((rows.size,), dtype=np.float64)
    sl = _slopes(alibi_slopes, Hq)
    rc = _load().oracle_attn_rows(_ptr(q, ctypes.c_float), _ptr(k, ctypes.c_float),
                                  _ptr(v, ctypes.c_float), _ptr(o, ctypes.c_double),
                                  _ptr(lse, ctypes.c_double), B, Hq, Hkv, Nq, Nk, d,
                                  float(scale), int(bool(causal)), int(window), _sp(sl),
                                  _ptr(rows, ctypes.c_int64), int(rows.size),
                                  int(nthreads or max_threads()))
    if rc != 0:
        raise ValueError("oracle_attn_rows failed with code %d" % rc)
    return o, lse


def prefill_paged(q, k_pages_bf16_bits, v_pages_bf16_bits, block_table, seq_lens, cu_q,
                  scale: float, nthreads: int | None = None):
    """Chunked prefill over a paged cache in fp64.

    q [T,Hq,d] (float32 values, token-major; sequence s owns rows
    cu_q[s]..cu_q[s+1]-1, the last cu_q[s+1]-cu_q[s] of its seq_lens[s]
    positions); pages [num_pages,Hkv,page_size,d] as bf16 bit patterns.
    Returns (O [T,Hq,d], L [T,Hq]) in float64.
    """
    q = _f32(q)
    kp = np.ascontiguousarray(np.asarray(k_pages_bf16_bits, dtype=np.uint16))
    vp = np.ascontiguousarray(np.asarray(v_pages_bf16_bits, dtype=np.uint16))
    bt = np.ascontiguousarray(np.asarray(block_table, dtype=np.int32))
    sl = np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int32))
    cq = np.ascontiguousarray(np.asarray(cu_q, dtype=np.int32))
    T, Hq, d = q.shape
    num_pages, Hkv, page_size, d2 = kp.shape
    S = sl.size
    if d2 != d or vp.shape != kp.shape or cq.size != S + 1 or int(cq[-1]) != T:
        raise ValueError("shape mismatch")
    _table_dims(S, bt, sl)
    o = np.zeros((T, Hq, d), dtype=np.float64)
    lse = np.zeros((T, Hq), dtype=np.float64)
    rc = _load().oracle_prefill_paged(_ptr(q, ctypes.c_float), _ptr(kp, ctypes.c_uint16),
                                      _ptr(vp, ctypes.c_uint16), _ptr(bt, ctypes.c_int32),
                                      _ptr(sl, ctypes.c_int32), _ptr(cq, ctypes.c_int32),
                                      _ptr(o, ctypes.c_double), _ptr(lse, ctypes.c_double),
                                      S, Hq, Hkv, d, page_size, bt.shape[1], num_pages,
                                      float(scale), int(nthreads or max_threads()))
    if rc != 0:
        raise ValueError("oracle_prefill_paged failed with code %d" % rc)
    return o, lse


def attention_bwd(q, k, v, do, scale: float, causal: bool = False, window: int = 0,
                  alibi_slopes=None, nthreads: int | None = None):
    """Gradients of attention in fp64: q, do [B,Hq,N,d], k, v [B,Hkv,N,d].

    Returns (dQ [B,Hq,N,d], dK [B,Hkv,N,d], dV [B,Hkv,N,d]) in float64, the
    derivatives of sum(do * O) with O = attention(q, k, v, ...).
    """
    q, k, v, do = _f32(q), _f32(k), _f32(v), _f32(do)
    B, Hq, Hkv, N, N2, d = _qkv_dims(q, k, v, do)
    if N2 != N:
        raise ValueError("shape mismatch")
    dq = np.zeros((B, Hq, N, d), dtype=np.float64)
    dk = np.zeros((B, Hkv, N, d), dtype=np.float64)
    dv = np.zeros((B, Hkv, N, d), dtype=np.float64)
    sl = _slopes(alibi_slopes, Hq)
    rc = _load().oracle_attn_bwd(_ptr(q, ctypes.c_float), _ptr(k, ctypes.c_float),
                                 _ptr(v, ctypes.c_float), _ptr(do, ctypes.c_float),
                                 _ptr(dq, ctypes.c_double), _ptr(dk, ctypes.c_double),
                                 _ptr(dv, ctypes.c_double), B, Hq, Hkv, N, d, float(scale),
                                 int(bool(causal)), int(window), _sp(sl),
                                 int(nthreads or max_threads()))
    if rc != 0:
        raise ValueError("oracle_attn_bwd failed with code %d" % rc)
    return dq, dk, dv


def attention_bwd_dq_rows(q, k, v, do, scale: float, causal: bool, rows, window: int = 0,
                          alibi_slopes=None, nthreads: int | None = None):
    """dQ of selected rows; rows[r] = (b*Hq + h)*N + i.  Returns [len(rows), d]."""
    q, k, v, do = _f32(q), _f32(k), _f32(v), _f32(do)
    B, Hq, Hkv, N, N2, d = _qkv_dims(q, k, v, do)
    if N2 != N:
        raise ValueError("shape mismatch")
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    out = np.zeros((rows.size, d), dtype=np.float64)
    sl = _slopes(alibi_slopes, Hq)
    rc = _load().oracle_attn_bwd_dq_rows(_ptr(q, ctypes.c_float), _ptr(k, ctypes.c_float),
                                         _ptr(v, ctypes.c_float), _ptr(do, ctypes.c_float),
                                         _ptr(out, ctypes.c_double), B, Hq, Hkv, N, d,
                                         float(scale), int(bool(causal)), int(window), _sp(sl),
                                         _ptr(rows, ctypes.c_int64), int(rows.size),
                                         int(nthreads or max_threads()))
    if rc != 0:
        raise ValueError("oracle_attn_bwd_dq_rows failed with code %d" % rc)
    return out


def attention_bwd_dkv_rows(q, k, v, do, scale: float, causal: bool, keys, window: int = 0,
                           alibi_slopes=None, nthreads: int | None = None):
    """dK and dV of selected keys; keys[r] = (b*Hkv + g)*N + j.  Returns two [len(keys), d]."""
    q, k, v, do = _f32(q), _f32(k), _f32(v), _f32(do)
    B, Hq, Hkv, N, N2, d = _qkv_dims(q, k, v, do)
    if N2 != N:
        raise ValueError("shape mismatch")
    keys = np.ascontiguousarray(np.asarray(keys, dtype=np.int64))
    dk = np.zeros((keys.size, d), dtype=np.float64)
    dv = np.zeros((keys.size, d), dtype=np.float64)
    sl = _slopes(alibi_slopes, Hq)
    rc = _load().oracle_attn_bwd_dkv_rows(_ptr(q, ctypes.c_float), _ptr(k, ctypes.c_float),
                                          _ptr(v, ctypes.c_float), _ptr(do, ctypes.c_float),
                                          _ptr(dk, ctypes.c_double), _ptr(dv, ctypes.c_double),
                                          B, Hq, Hkv, N, d, float(scale), int(bool(causal)),
                                          int(window), _sp(sl), _ptr(keys, ctypes.c_int64),
                                          int(keys.size), int(nthreads or max_threads()))
    if rc != 0:
        raise ValueError("oracle_attn_bwd_dkv_rows failed with code %d" % rc)
    return dk, dv


def decode_paged(q, k_pages_bf16_bits, v_pages_bf16_bits, block_table, seq_lens,
                 scale: float, seq_ids=None, nthreads: int | None = None):
    """Single-token paged decode in fp64 for the sequences in seq_ids.

    q [S,Hq,d] float32 values; k/v pages [num_pages,Hkv,page_size,d] as uint16
    bf16 bit patterns; block_table [S,max_blocks] int32; seq_lens [S] int32.
    Returns (O [nseq,Hq,d], L [nseq,Hq]) in float64.
    """
    q = _f32(q)
    kp = np.ascontiguousarray(np.asarray(k_pages_bf16_bits, dtype=np.uint16))
    vp = np.ascontiguousarray(np.asarray(v_pages_bf16_bits, dtype=np.uint16))
    bt = np.ascontiguousarray(np.asarray(block_table, dtype=np.int32))
    sl = np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int32))
    S, Hq, d = q.shape
    num_pages, Hkv, page_size, d2 = kp.shape
    if d2 != d or vp.shape != kp.shape:
        raise ValueError("page pool shape mismatch")
    _table_dims(S, bt, sl)
    max_blocks = bt.shape[1]
    if seq_ids is None:
        seq_ids = np.arange(S, dtype=np.int32)
    seq_ids = np.ascontiguousarray(np.asarray(seq_ids, dtype=np.int32))
    o = np.zeros((seq_ids.size, Hq, d), dtype=np.float64)
    lse = np.zeros((seq_ids.size, Hq), dtype=np.float64)
    rc = _load().oracle_decode_paged(_ptr(q, ctypes.c_float), _ptr(kp, ctypes.c_uint16),
                                     _ptr(vp, ctypes.c_uint16), _ptr(bt, ctypes.c_int32),
                                     _ptr(sl, ctypes.c_int32), _ptr(o, ctypes.c_double),
                                     _ptr(lse, ctypes.c_double), S, Hq, Hkv, d, page_size,
                                     max_blocks, num_pages, float(scale),
                                     _ptr(seq_ids, ctypes.c_int32), int(seq_ids.size),
                                     int(nthreads or max_threads()))
    if rc != 0:
        raise ValueError("oracle_decode_paged failed with code %d" % rc)
    return o, lse


def e4m3_to_double(byte: int) -> float:
    """The oracle's decoding of one FP8 E4M3 byte."""
    return float(_load().oracle_e4m3_to_double(int(byte)))


KV_FORMATS = {"e4m3": 0, "int8": 1}


def _bytes(a) -> np.ndarray:
    a = np.asarray(a)
    return np.ascontiguousarray(a.view(np.uint8) if a.dtype == np.int8 else a.astype(np.uint8, copy=False))


def decode_paged_q8(q, k_pages_u8, v_pages_u8, k_scales, v_scales, block_table, seq_lens,
                    scale: float, fmt: str = "e4m3", seq_ids=None, nthreads: int | None = None):
    """Decode over an 8-bit paged cache with one scale per (page, kv head).

    k/v pages [num_pages,Hkv,page_size,d] uint8 holding E4M3 (fmt "e4m3") or
    two's-complement INT8 (fmt "int8") bytes; k/v scales [num_pages,Hkv]
    float32; element = scale * decoded byte.  Returns (O [nseq,Hq,d],
    L [nseq,Hq]) in float64.
    """
    q = _f32(q)
    kp, vp = _bytes(k_pages_u8), _bytes(v_pages_u8)
    ks = _f32(k_scales)
    vs = _f32(v_scales)
    bt = np.ascontiguousarray(np.asarray(block_table, dtype=np.int32))
    sl = np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int32))
    S, Hq, d = q.shape
    num_pages, Hkv, page_size, d2 = kp.shape
    if d2 != d or vp.shape != kp.shape or ks.shape != (num_pages, Hkv) or vs.shape != ks.shape:
        raise ValueError("page pool / scale shape mismatch")
    _table_dims(S, bt, sl)
    max_blocks = bt.shape[1]
    if seq_ids is None:
        seq_ids = np.arange(S, dtype=np.int32)
    seq_ids = np.ascontiguousarray(np.asarray(seq_ids, dtype=np.int32))
    o = np.zeros((seq_ids.size, Hq, d), dtype=np.float64)
    lse = np.zeros((seq_ids.size, Hq), dtype=np.float64)
    rc = _load().oracle_decode_paged_q8(
        _ptr(q, ctypes.c_float), _ptr(kp, ctypes.c_uint8), _ptr(vp, ctypes.c_uint8),
        _ptr(ks, ctypes.c_float), _ptr(vs, ctypes.c_float), _ptr(bt, ctypes.c_int32),
        _ptr(sl, ctypes.c_int32), _ptr(o, ctypes.c_double), _ptr(lse, ctypes.c_double),
        S, Hq, Hkv, d, page_size, max_blocks, num_pages, float(scale), KV_FORMATS[fmt],
        _ptr(seq_ids, ctypes.c_int32), int(seq_ids.size), int(nthreads or max_threads()))
    if rc != 0:
        raise ValueError("oracle_decode_paged_q8 failed with code %d" % rc)
    return o, lse
