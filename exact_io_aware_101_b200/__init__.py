"""exact_io_aware_101_b200 -- exact, IO-aware attention on NVIDIA B200 (sm_100a).

A thin ctypes binding over ``libexattn.so`` (C ABI in ``include/exattn.h``).
Every step of the computation runs in the library's CUDA kernels; this module
only checks tensors, allocates outputs with PyTorch and passes device pointers
and the current CUDA stream.  There is no fallback: if the library is missing
or the device is not sm_100, calls raise.

    o, lse = attn_fwd(q, k, v, causal=True)                  # bf16 prefill
    o, lse = attn_fwd_f32(q, k, v)                           # fp32 prefill
    o, lse = attn_decode_paged(q, k_pages, v_pages, block_table, seq_lens)

Device-side failures (a corrupt block table, a bounded wait that ran out) are
reported as ATTN_DEV_* bits: a decode given a ``workspace`` reports into that
workspace (``decode_read_status``), every other call into the device's word
(``device_status``).
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

__all__ = [
    "attn_fwd", "attn_fwd_f32", "attn_decode_paged", "attn_decode_paged_noalloc",
    "attn_decode_paged_q8", "KV_FORMATS", "decode_workspace_bytes", "attn_bwd",
    "attn_prefill_paged",
    "bwd_workspace_bytes", "DECODE_NOALLOC_SCRATCH_BYTES",
    "device_status", "decode_read_status", "status_string", "version", "library", "LIB_PATH", "EXPORTED_SYMBOLS",
    "ATTN_DEV_BAD_PAGE", "ATTN_DEV_TIMEOUT", "ATTN_DEV_LAYOUT", "AttnError",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libexattn.so")
EXPORTED_SYMBOLS = ("attn_fwd", "attn_fwd_f32", "attn_fwd_ext", "attn_fwd_f32_ext",
                    "attn_bwd_workspace_bytes", "attn_bwd", "attn_prefill_paged",
                    "attn_decode_workspace_bytes",
                    "attn_decode_paged", "attn_decode_paged_noalloc", "attn_decode_paged_q8",
                    "attn_decode_read_status", "attn_device_status",
                    "attn_status_string", "attn_version")
# Size of the library's fixed per-device scratch used by attn_decode_paged_noalloc.
DECODE_NOALLOC_SCRATCH_BYTES = 32 << 20
ATTN_DEV_BAD_PAGE = 0x1
ATTN_DEV_TIMEOUT = 0x2
ATTN_DEV_LAYOUT = 0x4
# kv_format codes of attn_decode_paged_q8 and the torch dtypes accepted for each.
KV_FORMATS = {"e4m3": 0, "int8": 1}
_KV_DTYPES = {"e4m3": (torch.float8_e4m3fn, torch.uint8), "int8": (torch.int8,)}
_STATUS = {0: "ATTN_OK", 1: "ATTN_ERR_INVALID_ARG", 2: "ATTN_ERR_UNSUPPORTED", 3: "ATTN_ERR_CUDA"}

_lib = None


class AttnError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__("%s failed: %s" % (what, _STATUS.get(code, "status %d" % code)))
        self.code = code


def load_library(path: str) -> ctypes.CDLL:
    """Load a build of the C ABI at ``path`` and declare every entry point's types."""
    if not os.path.exists(path):
        raise ImportError("%s is not built; run `python -m exact_io_aware_101_b200.build`" % path)
    lib = ctypes.CDLL(path)
    _declare(lib)
    return lib


def library() -> ctypes.CDLL:
    """Load libexattn.so (built by ``python -m exact_io_aware_101_b200.build``)."""
    global _lib
    if _lib is None:
        _lib = load_library(LIB_PATH)
    return _lib


def _declare(lib: ctypes.CDLL) -> None:
    vp, ci, cf = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.attn_fwd.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, cf, ci, vp]
    lib.attn_fwd.restype = ci
    lib.attn_fwd_f32.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, cf, ci, vp]
    lib.attn_fwd_f32.restype = ci
    lib.attn_fwd_ext.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, cf, ci, ci, vp, vp]
    lib.attn_fwd_ext.restype = ci
    lib.attn_fwd_f32_ext.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, cf, ci, ci, vp, vp]
    lib.attn_fwd_f32_ext.restype = ci
    lib.attn_prefill_paged.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci,
                                       ci, ci, ci, cf, ci, vp, vp]
    lib.attn_prefill_paged.restype = ci
    lib.attn_bwd_workspace_bytes.argtypes = [ci, ci, ci]
    lib.attn_bwd_workspace_bytes.restype = ctypes.c_size_t
    lib.attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, cf, ci, ci,
                             vp, vp, ctypes.c_size_t, vp]
    lib.attn_bwd.restype = ci
    lib.attn_decode_workspace_bytes.argtypes = [ci, ci, ci, ci, ci]
    lib.attn_decode_workspace_bytes.restype = ctypes.c_size_t
    lib.attn_decode_paged.argtypes = [vp, vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, ci,
                                      cf, vp, ctypes.c_size_t, vp]
    lib.attn_decode_paged.restype = ci
    lib.attn_decode_paged_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, ci,
                                              ci, ci, cf, vp]
    lib.attn_decode_paged_noalloc.restype = ci
    lib.attn_decode_paged_q8.argtypes = [vp, vp, vp, vp, vp, ci, vp, vp, vp, vp, ci, ci, ci,
                                         ci, ci, ci, ci, cf, vp, ctypes.c_size_t, vp]
    lib.attn_decode_paged_q8.restype = ci
    lib.attn_decode_read_status.argtypes = [vp, ctypes.POINTER(ctypes.c_uint)]
    lib.attn_decode_read_status.restype = ci
    lib.attn_device_status.argtypes = [ctypes.POINTER(ctypes.c_uint), ci, vp]
    lib.attn_device_status.restype = ci
    lib.attn_status_string.argtypes = [ci]
    lib.attn_status_string.restype = ctypes.c_char_p
    lib.attn_version.argtypes = []
    lib.attn_version.restype = ctypes.c_char_p


def status_string(code: int) -> str:
    return library().attn_status_string(int(code)).decode()


def version() -> str:
    return library().attn_version().decode()


def _stream(t: torch.Tensor) -> int:
    return torch.cuda.current_stream(t.device).cuda_stream


def _check(t: torch.Tensor, name: str, dtype, ndim: int):
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % name)
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if t.dim() != ndim:
        raise ValueError("%s must have %d dims, got shape %s" % (name, ndim, tuple(t.shape)))
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


def _dims(t, name: str, ndim: int):
    """Type and rank of one argument, checked before its dtype or device so that
    shape errors are reported the same way on any device."""
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % name)
    if t.dim() != ndim:
        raise ValueError("%s must have %d dims, got shape %s" % (name, ndim, tuple(t.shape)))


def _same_device(device, **tensors):
    """Every tensor of one call must live on the device the call runs on: the
    kernel is launched there, and another GPU's pointer is not valid in it."""
    for name, t in tensors.items():
        if t is not None and t.device != device:
            raise ValueError("%s is on %s but q is on %s" % (name, t.device, device))


def _raise(rc: int, what: str):
    if rc != 0:
        raise AttnError(rc, what)


def _prefill(fn, what, q, k, v, causal, scale, out, lse, dtype, window=0, alibi_slopes=None):
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _dims(t, n, 4)
    B, Hq, N, d = q.shape
    if k.shape != v.shape or k.shape[0] != B or k.shape[2] != N or k.shape[3] != d:
        raise ValueError("k/v must be [B, Hkv, N, d] matching q %s" % (tuple(q.shape),))
    Hkv = k.shape[1]
    if out is not None:
        _dims(out, "out", 4)
    if lse is not None:
        _dims(lse, "lse", 3)
    if (out is not None and tuple(out.shape) != tuple(q.shape)) or \
            (lse is not None and tuple(lse.shape) != (B, Hq, N)):
        raise ValueError("out/lse shapes do not match q")
    if alibi_slopes is not None:
        _dims(alibi_slopes, "alibi_slopes", 1)
        if alibi_slopes.numel() != Hq:
            raise ValueError("alibi_slopes needs one value per query head")
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check(t, n, dtype, 4)
    _same_device(q.device, k=k, v=v, out=out, lse=lse, alibi_slopes=alibi_slopes)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    _check(out, "out", dtype, 4)
    _check(lse, "lse", torch.float32, 3)
    if tuple(out.shape) != tuple(q.shape) or tuple(lse.shape) != (B, Hq, N):
        raise ValueError("out/lse shapes do not match q")
    if window or alibi_slopes is not None:
        slopes_ptr = None
        if alibi_slopes is not None:
            _check(alibi_slopes, "alibi_slopes", torch.float32, 1)
            slopes_ptr = alibi_slopes.data_ptr()
        ext = getattr(library(), fn.__name__ + "_ext")
        with torch.cuda.device(q.device):
            rc = ext(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                     B, Hq, Hkv, N, d, float(scale), int(bool(causal)), int(window), slopes_ptr,
                     _stream(q))
    else:
        with torch.cuda.device(q.device):
            rc = fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                    B, Hq, Hkv, N, d, float(scale), int(bool(causal)), _stream(q))
    _raise(rc, what)
    return out, lse


def attn_fwd(q, k, v, causal: bool = False, scale: float | None = None, out=None, lse=None,
             window: int = 0, alibi_slopes=None):
    """bf16 prefill: q [B,Hq,N,d], k/v [B,Hkv,N,d] -> (O bf16 [B,Hq,N,d], L fp32 [B,Hq,N]).

    window > 0 (with causal): keys with i - j >= window are masked.  alibi_slopes:
    a CUDA float32 tensor [Hq]; slope_h * (j - i) is added to the scaled scores.
    """
    return _prefill(library().attn_fwd, "attn_fwd", q, k, v, causal, scale, out, lse,
                    torch.bfloat16, window, alibi_slopes)


def attn_fwd_f32(q, k, v, causal: bool = False, scale: float | None = None, out=None, lse=None,
                 window: int = 0, alibi_slopes=None):
    """fp32 prefill with fp32 arithmetic throughout (same options as attn_fwd)."""
    return _prefill(library().attn_fwd_f32, "attn_fwd_f32", q, k, v, causal, scale, out, lse,
                    torch.float32, window, alibi_slopes)


def attn_prefill_paged(q, k_pages, v_pages, block_table, seq_lens, cu_q, max_q: int,
                       scale: float | None = None, window: int = 0, alibi_slopes=None,
                       out=None, lse=None):
    """Chunked prefill over the paged cache.

    q [T,Hq,d] bf16 token-major (sequence s: rows cu_q[s]..cu_q[s+1]-1, the
    last tokens of its seq_lens[s]); pages [num_pages,Hkv,16,d] bf16;
    block_table [S,max_blocks], seq_lens [S], cu_q [S+1] int32 (GPU).  max_q
    bounds every chunk length.  Returns (O bf16 [T,Hq,d], L fp32 [T,Hq]).
    """
    for name, t, nd in (("q", q, 3), ("k_pages", k_pages, 4), ("v_pages", v_pages, 4),
                        ("block_table", block_table, 2), ("seq_lens", seq_lens, 1),
                        ("cu_q", cu_q, 1)):
        _dims(t, name, nd)
    T, Hq, d = q.shape
    num_pages, Hkv, page_size, d2 = k_pages.shape
    S = seq_lens.shape[0]
    if d2 != d or tuple(v_pages.shape) != tuple(k_pages.shape):
        raise ValueError("page pools must be [num_pages, Hkv, page_size, d]")
    if block_table.shape[0] != S or cu_q.shape[0] != S + 1:
        raise ValueError("block_table needs S rows and cu_q S+1 entries")
    if out is not None:
        _dims(out, "out", 3)
    if lse is not None:
        _dims(lse, "lse", 2)
    if (out is not None and tuple(out.shape) != tuple(q.shape)) or \
            (lse is not None and tuple(lse.shape) != (T, Hq)):
        raise ValueError("out must be [T, Hq, d] and lse [T, Hq]")
    if alibi_slopes is not None:
        _dims(alibi_slopes, "alibi_slopes", 1)
        if alibi_slopes.numel() != Hq:
            raise ValueError("alibi_slopes needs one value per query head")
    _check(q, "q", torch.bfloat16, 3)
    _check(k_pages, "k_pages", torch.bfloat16, 4)
    _check(v_pages, "v_pages", torch.bfloat16, 4)
    _check(block_table, "block_table", torch.int32, 2)
    _check(seq_lens, "seq_lens", torch.int32, 1)
    _check(cu_q, "cu_q", torch.int32, 1)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((T, Hq), dtype=torch.float32, device=q.device) if lse is None else lse
    _check(out, "out", torch.bfloat16, 3)
    _check(lse, "lse", torch.float32, 2)
    slopes_ptr = None
    if alibi_slopes is not None:
        _check(alibi_slopes, "alibi_slopes", torch.float32, 1)
        slopes_ptr = alibi_slopes.data_ptr()
    _same_device(q.device, k_pages=k_pages, v_pages=v_pages, block_table=block_table,
                 seq_lens=seq_lens, cu_q=cu_q, out=out, lse=lse, alibi_slopes=alibi_slopes)
    with torch.cuda.device(q.device):
        rc = library().attn_prefill_paged(q.data_ptr(), k_pages.data_ptr(), v_pages.data_ptr(),
                                          block_table.data_ptr(), seq_lens.data_ptr(),
                                          cu_q.data_ptr(), out.data_ptr(), lse.data_ptr(), S, Hq,
                                          Hkv, T, int(max_q), d, page_size, block_table.shape[1],
                                          num_pages, float(scale), int(window), slopes_ptr,
                                          _stream(q))
    _raise(rc, "attn_prefill_paged")
    return out, lse


def bwd_workspace_bytes(B: int, Hq: int, N: int) -> int:
    return int(library().attn_bwd_workspace_bytes(B, Hq, N))


def attn_bwd(q, k, v, o, lse, dout, causal: bool = False, scale: float | None = None,
             window: int = 0, alibi_slopes=None, dq=None, dk=None, dv=None, workspace=None):
    """Gradients (dQ, dK, dV) of sum(dout * O) for the bf16 attention.

    q, o, dout [B,Hq,N,d] bf16; k, v [B,Hkv,N,d] bf16; lse [B,Hq,N] fp32 as
    attn_fwd returned them for the same inputs and options.  Returns bf16
    (dQ [B,Hq,N,d], dK [B,Hkv,N,d], dV [B,Hkv,N,d]).
    """
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout)):
        _dims(t, name, 4)
    _dims(lse, "lse", 3)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    if tuple(o.shape) != tuple(q.shape) or tuple(dout.shape) != tuple(q.shape):
        raise ValueError("o and dout must have q's shape")
    if tuple(k.shape) != (B, Hkv, N, d) or tuple(v.shape) != tuple(k.shape):
        raise ValueError("k and v must be [B, Hkv, N, d]")
    if tuple(lse.shape) != (B, Hq, N):
        raise ValueError("lse must be [B, Hq, N]")
    for name, t, like in (("dq", dq, q), ("dk", dk, k), ("dv", dv, v)):
        if t is not None:
            _dims(t, name, 4)
            if tuple(t.shape) != tuple(like.shape):
                raise ValueError("dq must have q's shape, dk and dv k's shape")
    for name, t in (("q", q), ("o", o), ("dout", dout)):
        _check(t, name, torch.bfloat16, 4)
    _check(k, "k", torch.bfloat16, 4)
    _check(v, "v", torch.bfloat16, 4)
    _check(lse, "lse", torch.float32, 3)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _check(dq, "dq", torch.bfloat16, 4)
    _check(dk, "dk", torch.bfloat16, 4)
    _check(dv, "dv", torch.bfloat16, 4)
    slopes_ptr = None
    if alibi_slopes is not None:
        alibi_slopes = torch.as_tensor(alibi_slopes, dtype=torch.float32, device=q.device).contiguous()
        if alibi_slopes.numel() != Hq:
            raise ValueError("need one ALiBi slope per query head")
        slopes_ptr = alibi_slopes.data_ptr()
    need = bwd_workspace_bytes(B, Hq, N)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _check(workspace, "workspace", torch.uint8, 1)
    _same_device(q.device, k=k, v=v, o=o, lse=lse, dout=dout, dq=dq, dk=dk, dv=dv,
                 alibi_slopes=alibi_slopes, workspace=workspace)
    with torch.cuda.device(q.device):
        rc = library().attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                lse.data_ptr(), dout.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                                dv.data_ptr(), B, Hq, Hkv, N, d, float(scale), int(bool(causal)),
                                int(window), slopes_ptr, workspace.data_ptr(), workspace.numel(),
                                _stream(q))
    _raise(rc, "attn_bwd")
    return dq, dk, dv


def decode_workspace_bytes(S: int, Hq: int, d: int, max_blocks: int, page_size: int = 16) -> int:
    return int(library().attn_decode_workspace_bytes(S, Hq, d, max_blocks, page_size))


def _decode_dims(q, k_pages, v_pages, block_table, seq_lens):
    """Shapes of a paged decode's tensors, checked against one another before any
    dtype or device check: the library gets no tensor sizes, so a block_table or
    seq_lens with fewer than S rows would be read past its end on the device."""
    for name, t, nd in (("q", q, 3), ("k_pages", k_pages, 4), ("v_pages", v_pages, 4),
                        ("block_table", block_table, 2), ("seq_lens", seq_lens, 1)):
        _dims(t, name, nd)
    S, Hq, d = q.shape
    num_pages, Hkv, page_size, d2 = k_pages.shape
    if d2 != d or tuple(v_pages.shape) != tuple(k_pages.shape):
        raise ValueError("page pools must be [num_pages, Hkv, page_size, d] with q's d, and "
                         "v_pages must match k_pages")
    if block_table.shape[0] != S or seq_lens.shape[0] != S:
        raise ValueError("block_table/seq_lens must have S rows")
    return S, Hq, d, num_pages, Hkv, page_size, block_table.shape[1]


def _decode_out_dims(q, S, Hq, out, lse):
    """Caller-given outputs of a decode, checked for shape before any device check."""
    if out is not None:
        _dims(out, "out", 3)
    if lse is not None:
        _dims(lse, "lse", 2)
    if (out is not None and tuple(out.shape) != tuple(q.shape)) or \
            (lse is not None and tuple(lse.shape) != (S, Hq)):
        raise ValueError("out must be [S, Hq, d] and lse [S, Hq]")


def _decode_outputs(q, S, Hq, out, lse):
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((S, Hq), dtype=torch.float32, device=q.device)
    _check(out, "out", torch.bfloat16, 3)
    _check(lse, "lse", torch.float32, 2)
    if tuple(out.shape) != tuple(q.shape) or tuple(lse.shape) != (S, Hq):
        raise ValueError("out must be [S, Hq, d] and lse [S, Hq]")
    return out, lse


def attn_decode_paged(q, k_pages, v_pages, block_table, seq_lens, scale: float | None = None,
                      out=None, lse=None, workspace=None):
    """Paged single-token decode.

    q [S,Hq,d] bf16; k_pages/v_pages [num_pages,Hkv,page_size,d] bf16;
    block_table [S,max_blocks] int32; seq_lens [S] int32 (all on the GPU).
    Returns (O bf16 [S,Hq,d], L fp32 [S,Hq]).  ``workspace`` (uint8, at least
    decode_workspace_bytes(...) bytes) is allocated when not given; pass one to
    read the call's status afterwards with ``decode_read_status(workspace)``.
    """
    S, Hq, d, num_pages, Hkv, page_size, max_blocks = _decode_dims(q, k_pages, v_pages,
                                                                   block_table, seq_lens)
    _decode_out_dims(q, S, Hq, out, lse)
    _check(q, "q", torch.bfloat16, 3)
    _check(k_pages, "k_pages", torch.bfloat16, 4)
    _check(v_pages, "v_pages", torch.bfloat16, 4)
    _check(block_table, "block_table", torch.int32, 2)
    _check(seq_lens, "seq_lens", torch.int32, 1)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out, lse = _decode_outputs(q, S, Hq, out, lse)
    need = decode_workspace_bytes(S, Hq, d, max_blocks, page_size)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _check(workspace, "workspace", torch.uint8, 1)
    _same_device(q.device, k_pages=k_pages, v_pages=v_pages, block_table=block_table,
                 seq_lens=seq_lens, out=out, lse=lse, workspace=workspace)
    with torch.cuda.device(q.device):
        rc = library().attn_decode_paged(q.data_ptr(), k_pages.data_ptr(), v_pages.data_ptr(),
                                         block_table.data_ptr(), seq_lens.data_ptr(),
                                         out.data_ptr(), lse.data_ptr(), S, Hq, Hkv, d, page_size,
                                         max_blocks, num_pages, float(scale), workspace.data_ptr(),
                                         workspace.numel(), _stream(q))
    _raise(rc, "attn_decode_paged")
    return out, lse


def attn_decode_paged_q8(q, k_pages, v_pages, k_scales, v_scales, block_table, seq_lens,
                         kv_format: str = "e4m3", scale: float | None = None, out=None, lse=None,
                         workspace=None):
    """Paged single-token decode over an 8-bit KV cache.

    k_pages/v_pages [num_pages,Hkv,page_size,d]: E4M3 codes (torch.float8_e4m3fn,
    or their bytes as uint8) for kv_format "e4m3", torch.int8 for "int8";
    k_scales/v_scales [num_pages,Hkv] float32, one per (page, K/V head): the
    element is scale * code.  Everything else (the workspace and its status
    word included) as attn_decode_paged.
    """
    if kv_format not in KV_FORMATS:
        raise ValueError("kv_format must be one of %s" % sorted(KV_FORMATS))
    S, Hq, d, num_pages, Hkv, page_size, max_blocks = _decode_dims(q, k_pages, v_pages,
                                                                   block_table, seq_lens)
    _decode_out_dims(q, S, Hq, out, lse)
    for name, t in (("k_scales", k_scales), ("v_scales", v_scales)):
        _dims(t, name, 2)
        if tuple(t.shape) != (num_pages, Hkv):
            raise ValueError("scales must be [num_pages, Hkv]")
    _check(q, "q", torch.bfloat16, 3)
    for name, t in (("k_pages", k_pages), ("v_pages", v_pages)):
        if t.dtype not in _KV_DTYPES[kv_format]:
            raise TypeError("%s must be one of %s for kv_format %r"
                            % (name, _KV_DTYPES[kv_format], kv_format))
        _check(t, name, t.dtype, 4)
    _check(k_scales, "k_scales", torch.float32, 2)
    _check(v_scales, "v_scales", torch.float32, 2)
    _check(block_table, "block_table", torch.int32, 2)
    _check(seq_lens, "seq_lens", torch.int32, 1)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out, lse = _decode_outputs(q, S, Hq, out, lse)
    need = decode_workspace_bytes(S, Hq, d, max_blocks, page_size)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _check(workspace, "workspace", torch.uint8, 1)
    _same_device(q.device, k_pages=k_pages, v_pages=v_pages, k_scales=k_scales,
                 v_scales=v_scales, block_table=block_table, seq_lens=seq_lens, out=out, lse=lse,
                 workspace=workspace)
    with torch.cuda.device(q.device):
        rc = library().attn_decode_paged_q8(q.data_ptr(), k_pages.data_ptr(), v_pages.data_ptr(),
                                            k_scales.data_ptr(), v_scales.data_ptr(),
                                            KV_FORMATS[kv_format], block_table.data_ptr(),
                                            seq_lens.data_ptr(), out.data_ptr(), lse.data_ptr(), S,
                                            Hq, Hkv, d, page_size, max_blocks, num_pages,
                                            float(scale), workspace.data_ptr(), workspace.numel(),
                                            _stream(q))
    _raise(rc, "attn_decode_paged_q8")
    return out, lse


def attn_decode_paged_noalloc(q, k_pages, v_pages, block_table, seq_lens,
                              scale: float | None = None, out=None, lse=None):
    """Paged decode that allocates no device memory inside the library.

    For callers that may not call cudaMalloc (for example a plugin whose host
    program owns all device memory, or a decode loop that must not wait on the
    allocator): the chunk partials live in the library's fixed per-device scratch
    (DECODE_NOALLOC_SCRATCH_BYTES), shared by every such call on the device, so
    calls that overlap on the GPU race.  Pass ``out`` and ``lse`` to avoid torch
    allocating the outputs here.  Arguments as for attn_decode_paged; a bad page
    id or length is reported in the device's word (``device_status``).
    """
    S, Hq, d, num_pages, Hkv, page_size, max_blocks = _decode_dims(q, k_pages, v_pages,
                                                                   block_table, seq_lens)
    _decode_out_dims(q, S, Hq, out, lse)
    _check(q, "q", torch.bfloat16, 3)
    _check(k_pages, "k_pages", torch.bfloat16, 4)
    _check(v_pages, "v_pages", torch.bfloat16, 4)
    _check(block_table, "block_table", torch.int32, 2)
    _check(seq_lens, "seq_lens", torch.int32, 1)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out, lse = _decode_outputs(q, S, Hq, out, lse)
    _same_device(q.device, k_pages=k_pages, v_pages=v_pages, block_table=block_table,
                 seq_lens=seq_lens, out=out, lse=lse)
    with torch.cuda.device(q.device):
        rc = library().attn_decode_paged_noalloc(
            q.data_ptr(), k_pages.data_ptr(), v_pages.data_ptr(), block_table.data_ptr(),
            seq_lens.data_ptr(), out.data_ptr(), lse.data_ptr(), S, Hq, Hkv, d, page_size,
            max_blocks, num_pages, float(scale), _stream(q))
    _raise(rc, "attn_decode_paged_noalloc")
    return out, lse


def decode_read_status(workspace: torch.Tensor) -> int:
    """ATTN_DEV_* bits of the last workspace decode that used ``workspace`` (0: none).

    Synchronises nothing: first synchronise the stream the decode ran on (or an
    event recorded after it)."""
    _check(workspace, "workspace", torch.uint8, 1)
    st = ctypes.c_uint(0)
    with torch.cuda.device(workspace.device):
        rc = library().attn_decode_read_status(workspace.data_ptr(), ctypes.byref(st))
    _raise(rc, "attn_decode_read_status")
    return int(st.value)


def device_status(clear: bool = False, device=None) -> int:
    """Status bits (ATTN_DEV_*) that calls without a decode workspace raised on a device.

    Waits for the work enqueued so far on that device's current stream (and only
    for it)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    st = ctypes.c_uint(0)
    with torch.cuda.device(dev):
        rc = library().attn_device_status(ctypes.byref(st), int(bool(clear)),
                                          torch.cuda.current_stream(dev).cuda_stream)
    _raise(rc, "attn_device_status")
    return int(st.value)
