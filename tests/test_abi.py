"""The C ABI boundary on the CPU: the library loads, exports every entry point
that include/exattn.h declares, and rejects bad arguments before touching the
GPU.  No call here reaches a kernel launch."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

import exact_io_aware_101_b200 as ea  # noqa: E402
from exact_io_aware_101_b200 import build as eabuild  # noqa: E402

INVALID, UNSUPPORTED = 1, 2


@pytest.fixture(scope="module")
def lib():
    eabuild.build()
    return ea.library()


def declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(attn_[a-z0-9_]+)\s*\(", text))
    return names


def test_header_declares_the_boundary():
    names = declared_functions()
    assert {"attn_fwd", "attn_fwd_f32", "attn_decode_paged",
            "attn_decode_workspace_bytes"} <= names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(ea.EXPORTED_SYMBOLS) >= declared_functions()


def test_only_the_c_abi_is_exported(lib):
    # -fvisibility=hidden keeps internal C++ symbols out of the dynamic table.
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", ea.LIB_PATH], capture_output=True,
                         text=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    assert {s for s in exported if s.startswith("attn_")} == declared_functions()


def test_device_status_bits_match_the_header():
    text = open(os.path.join(ROOT, "include", "exattn.h")).read()
    bits = {name: int(val, 16) for name, val in
            re.findall(r"#define\s+(ATTN_DEV_[A-Z_]+)\s+(0x[0-9a-fA-F]+)u", text)}
    assert set(bits) == {"ATTN_DEV_BAD_PAGE", "ATTN_DEV_TIMEOUT", "ATTN_DEV_LAYOUT"}
    for name, val in bits.items():
        assert getattr(ea, name) == val, name
    assert len(set(bits.values())) == len(bits)  # distinct bits
    assert all(v & (v - 1) == 0 for v in bits.values())  # one bit each


def test_version_and_status_strings(lib):
    assert "sm_100a" in ea.version()
    assert ea.status_string(0) == "ATTN_OK"
    assert ea.status_string(1) == "ATTN_ERR_INVALID_ARG"
    assert ea.status_string(2) == "ATTN_ERR_UNSUPPORTED"
    assert ea.status_string(3) == "ATTN_ERR_CUDA"
    assert ea.status_string(99) == "ATTN_UNKNOWN_STATUS"


A = 1 << 20  # a fake, 16-byte-aligned address: validation fails before any use


def fwd(lib, q=A, k=A, v=A, o=A, lse=A, B=1, Hq=2, Hkv=1, N=16, d=128, scale=0.1, causal=0):
    return lib.attn_fwd(q, k, v, o, lse, B, Hq, Hkv, N, d, scale, causal, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), INVALID), (dict(o=A + 8), INVALID), (dict(lse=A + 2), INVALID),
    (dict(B=0), INVALID), (dict(N=0), INVALID), (dict(Hq=3, Hkv=2), INVALID),
    (dict(Hkv=0), INVALID), (dict(scale=float("nan")), INVALID), (dict(scale=-1.0), INVALID),
    (dict(scale=float("inf")), INVALID), (dict(scale=0.0), INVALID), (dict(d=96), UNSUPPORTED), (dict(d=256), UNSUPPORTED),
])
def test_prefill_argument_checks(lib, kw, code):
    assert fwd(lib, **kw) == code
    assert lib.attn_fwd_f32(*(kw.get(n, A) for n in ("q", "k", "v", "o", "lse")),
                            kw.get("B", 1), kw.get("Hq", 2), kw.get("Hkv", 1), kw.get("N", 16),
                            kw.get("d", 128), kw.get("scale", 0.1), 0, None) == code


@pytest.mark.parametrize("window,causal,slopes,code", [
    (-1, 1, None, INVALID), (8, 0, None, INVALID), (0, 1, A + 2, INVALID), (8, 1, A + 1, INVALID)])
def test_window_alibi_argument_checks(lib, window, causal, slopes, code):
    for fn in (lib.attn_fwd_ext, lib.attn_fwd_f32_ext):
        assert fn(A, A, A, A, A, 1, 2, 1, 16, 128, 0.1, causal, window, slopes, None) == code


def test_decode_workspace_size(lib):
    # 512 pages of 16 tokens in chunks of 32 pages -> 16 chunks per sequence;
    # a 256-byte status block precedes the partials.
    n = ea.decode_workspace_bytes(64, 32, 128, 512)
    parts = 64 * 32 * 16
    assert n >= 256 + parts * 129 * 4 and n % 256 == 0 and n < 256 + parts * 129 * 4 + 512
    assert ea.decode_workspace_bytes(64, 32, 96, 512) == 0
    assert ea.decode_workspace_bytes(64, 32, 128, 512, page_size=32) == 0
    assert ea.decode_workspace_bytes(0, 32, 128, 512) == 0


def dec(lib, ws_bytes=None, **kw):
    a = dict(q=A, kp=A, vp=A, bt=A, sl=A, o=A, lse=A, S=4, Hq=8, Hkv=2, d=128, ps=16, maxb=8,
             npages=100, scale=0.1, ws=A)
    a.update(kw)
    need = lib.attn_decode_workspace_bytes(a["S"], a["Hq"], a["d"], a["maxb"], 16) or 1 << 20
    return lib.attn_decode_paged(a["q"], a["kp"], a["vp"], a["bt"], a["sl"], a["o"], a["lse"],
                                 a["S"], a["Hq"], a["Hkv"], a["d"], a["ps"], a["maxb"],
                                 a["npages"], a["scale"], a["ws"],
                                 need if ws_bytes is None else ws_bytes, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), INVALID), (dict(ws=None), INVALID), (dict(kp=A + 4), INVALID),
    (dict(bt=A + 2), INVALID), (dict(S=0), INVALID), (dict(Hq=6, Hkv=4), INVALID),
    (dict(maxb=0), INVALID), (dict(npages=0), INVALID), (dict(scale=-0.5), INVALID),
    (dict(d=80), UNSUPPORTED), (dict(ps=8), UNSUPPORTED),
])
def test_decode_argument_checks(lib, kw, code):
    assert dec(lib, **kw) == code


def test_decode_rejects_small_workspace(lib):
    assert dec(lib, ws_bytes=64) == INVALID


def test_decode_read_status_argument_checks(lib):
    import ctypes
    st = ctypes.c_uint(7)
    assert lib.attn_decode_read_status(None, ctypes.byref(st)) == INVALID
    assert lib.attn_decode_read_status(A + 8, ctypes.byref(st)) == INVALID
    assert lib.attn_decode_read_status(A, None) == INVALID
    assert st.value == 7  # nothing written on an error
    assert lib.attn_device_status(None, 0, None) == INVALID


@pytest.mark.parametrize("which", ["paged", "q8", "noalloc"])
def test_decode_binding_checks_shapes_before_the_library(which):
    # The C side gets no tensor sizes, so the binding must reject a block table
    # or length vector with fewer rows than q has sequences, and pools that do
    # not agree, before any call (these CPU tensors never reach the library).
    import torch
    S, Hq, Hkv, d, P = 3, 8, 2, 128, 10
    q = torch.zeros(S, Hq, d, dtype=torch.bfloat16)
    kp = torch.zeros(P, Hkv, 16, d, dtype=torch.bfloat16)
    bt = torch.zeros(S, 4, dtype=torch.int32)
    sl = torch.zeros(S, dtype=torch.int32)
    sc = torch.ones(P, Hkv)

    def call(q=q, kp=kp, vp=kp, bt=bt, sl=sl):
        if which == "paged":
            return ea.attn_decode_paged(q, kp, vp, bt, sl)
        if which == "noalloc":
            return ea.attn_decode_paged_noalloc(q, kp, vp, bt, sl)
        return ea.attn_decode_paged_q8(q, kp.to(torch.int8), vp.to(torch.int8), sc, sc, bt, sl,
                                       kv_format="int8")
    with pytest.raises(ValueError, match="S rows"):
        call(bt=bt[:2])
    with pytest.raises(ValueError, match="S rows"):
        call(sl=sl[:1])
    with pytest.raises(ValueError, match="page pools"):
        call(vp=kp[:, :1].contiguous())
    with pytest.raises(ValueError, match="page pools"):
        call(q=torch.zeros(S, Hq, 64, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="dims"):
        call(bt=bt[0])


def test_python_binding_rejects_cpu_tensors():
    import torch
    q = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        ea.attn_fwd(q, q, q)
    with pytest.raises(TypeError):
        ea.attn_fwd(q.float(), q.float(), q.float())


def dec_q8(lib, ws_bytes=None, **kw):
    a = dict(q=A, kp=A, vp=A, ks=A, vs=A, fmt=0, bt=A, sl=A, o=A, lse=A, S=4, Hq=8, Hkv=2, d=128,
             ps=16, maxb=8, npages=100, scale=0.1, ws=A)
    a.update(kw)
    need = lib.attn_decode_workspace_bytes(a["S"], a["Hq"], a["d"], a["maxb"], 16) or 1 << 20
    return lib.attn_decode_paged_q8(a["q"], a["kp"], a["vp"], a["ks"], a["vs"], a["fmt"], a["bt"],
                                    a["sl"], a["o"], a["lse"], a["S"], a["Hq"], a["Hkv"], a["d"],
                                    a["ps"], a["maxb"], a["npages"], a["scale"], a["ws"],
                                    need if ws_bytes is None else ws_bytes, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), INVALID), (dict(ks=None), INVALID), (dict(vs=A + 2), INVALID),
    (dict(fmt=2), INVALID), (dict(fmt=-1), INVALID), (dict(S=0), INVALID),
    (dict(Hq=6, Hkv=4), INVALID), (dict(npages=0), INVALID), (dict(scale=float("nan")), INVALID),
    (dict(d=96), UNSUPPORTED), (dict(ps=32), UNSUPPORTED),
])
def test_decode_q8_argument_checks(lib, kw, code):
    assert dec_q8(lib, **kw) == code


def test_decode_q8_rejects_small_workspace(lib):
    assert dec_q8(lib, ws_bytes=64) == INVALID


def test_decode_noalloc_argument_checks(lib):
    def call(**kw):
        a = dict(q=A, kp=A, vp=A, bt=A, sl=A, o=A, lse=A, S=4, Hq=8, Hkv=2, d=128, ps=16, maxb=8,
                 npages=100, scale=0.1)
        a.update(kw)
        return lib.attn_decode_paged_noalloc(a["q"], a["kp"], a["vp"], a["bt"], a["sl"], a["o"],
                                             a["lse"], a["S"], a["Hq"], a["Hkv"], a["d"], a["ps"],
                                             a["maxb"], a["npages"], a["scale"], None)
    assert call(q=None) == INVALID
    assert call(Hq=6, Hkv=4) == INVALID
    assert call(d=80) == UNSUPPORTED
    # More partials than the fixed scratch holds.
    assert call(S=4096, Hq=64, maxb=4096) == INVALID


def paged(lib, **kw):
    a = dict(q=A, kp=A, vp=A, bt=A, sl=A, cu=A, o=A, lse=A, S=2, Hq=8, Hkv=2, T=64, maxq=32,
             d=128, ps=16, maxb=8, npages=100, scale=0.1, window=0, slopes=None)
    a.update(kw)
    return lib.attn_prefill_paged(a["q"], a["kp"], a["vp"], a["bt"], a["sl"], a["cu"], a["o"],
                                  a["lse"], a["S"], a["Hq"], a["Hkv"], a["T"], a["maxq"], a["d"],
                                  a["ps"], a["maxb"], a["npages"], a["scale"], a["window"],
                                  a["slopes"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), INVALID), (dict(cu=A + 2), INVALID), (dict(o=A + 8), INVALID),
    (dict(slopes=A + 1), INVALID), (dict(S=0), INVALID), (dict(Hq=6, Hkv=4), INVALID),
    (dict(T=-1), INVALID), (dict(maxq=-1), INVALID), (dict(window=-1), INVALID),
    (dict(scale=0.0), INVALID), (dict(d=96), UNSUPPORTED), (dict(ps=32), UNSUPPORTED),
])
def test_prefill_paged_argument_checks(lib, kw, code):
    assert paged(lib, **kw) == code


def test_prefill_paged_empty_is_a_no_op(lib):
    # Nothing to compute: no device is touched.
    assert paged(lib, T=0) == 0
    assert paged(lib, maxq=0) == 0


def test_bwd_workspace_size(lib):
    # L*log2(e) and D, each [B*Hq][N padded to 128] fp32, each 256-byte aligned.
    n = lib.attn_bwd_workspace_bytes(2, 16, 1000)
    rows = 2 * 16 * 1024
    assert n == 2 * ((rows * 4 + 255) // 256 * 256)
    assert lib.attn_bwd_workspace_bytes(0, 16, 1000) == 0
    assert lib.attn_bwd_workspace_bytes(2, 16, 0) == 0


def bwd(lib, ws_bytes=None, **kw):
    a = dict(q=A, k=A, v=A, o=A, lse=A, do=A, dq=A, dk=A, dv=A, B=1, Hq=2, Hkv=1, N=16, d=128,
             scale=0.1, causal=0, window=0, slopes=None, ws=A)
    a.update(kw)
    need = lib.attn_bwd_workspace_bytes(a["B"], a["Hq"], max(a["N"], 1)) or 1 << 20
    return lib.attn_bwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["do"], a["dq"], a["dk"],
                        a["dv"], a["B"], a["Hq"], a["Hkv"], a["N"], a["d"], a["scale"], a["causal"],
                        a["window"], a["slopes"], a["ws"], need if ws_bytes is None else ws_bytes,
                        None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), INVALID), (dict(do=None), INVALID), (dict(dk=A + 8), INVALID),
    (dict(ws=A + 4), INVALID), (dict(window=8, causal=0), INVALID), (dict(window=-1), INVALID),
    (dict(slopes=A + 2), INVALID), (dict(N=0), INVALID), (dict(Hq=3, Hkv=2), INVALID),
    (dict(scale=-1.0), INVALID), (dict(d=96), UNSUPPORTED),
])
def test_bwd_argument_checks(lib, kw, code):
    assert bwd(lib, **kw) == code


def test_bwd_rejects_small_workspace(lib):
    assert bwd(lib, ws_bytes=64) == INVALID


def test_binding_checks_output_shapes_before_the_library():
    # Caller-given outputs and gradients are written by the kernels at the sizes
    # the inputs imply, so a smaller tensor must be refused before any call
    # (these CPU tensors never reach the library).
    import torch
    bf = torch.bfloat16
    B, Hq, Hkv, N, d = 1, 4, 2, 8, 64
    q = torch.zeros(B, Hq, N, d, dtype=bf)
    k = torch.zeros(B, Hkv, N, d, dtype=bf)
    lse = torch.zeros(B, Hq, N)
    with pytest.raises(ValueError, match="out/lse shapes"):
        ea.attn_fwd(q, k, k, out=q[:, :2].contiguous())
    with pytest.raises(ValueError, match="out/lse shapes"):
        ea.attn_fwd(q, k, k, lse=lse[:, :, :4].contiguous())
    with pytest.raises(ValueError, match="one value per query head"):
        ea.attn_fwd(q, k, k, causal=True, alibi_slopes=torch.zeros(Hq - 1))
    with pytest.raises(ValueError, match="out/lse shapes"):
        ea.attn_fwd_f32(q.float(), k.float(), k.float(), out=q.float()[:, :, :4].contiguous())

    with pytest.raises(ValueError, match="dq must have"):
        ea.attn_bwd(q, k, k, q, lse, q, dq=q[:, :2].contiguous())
    with pytest.raises(ValueError, match="dq must have"):
        ea.attn_bwd(q, k, k, q, lse, q, dk=q)
    with pytest.raises(ValueError, match="dq must have"):
        ea.attn_bwd(q, k, k, q, lse, q, dv=k[:, :, :4].contiguous())

    S, P, T = 2, 6, 5
    qp = torch.zeros(T, Hq, d, dtype=bf)
    kp = torch.zeros(P, Hkv, 16, d, dtype=bf)
    bt = torch.zeros(S, 3, dtype=torch.int32)
    sl = torch.zeros(S, dtype=torch.int32)
    cu = torch.zeros(S + 1, dtype=torch.int32)
    with pytest.raises(ValueError, match=r"out must be \[T, Hq, d\]"):
        ea.attn_prefill_paged(qp, kp, kp, bt, sl, cu, 4, out=qp[:4].contiguous())
    with pytest.raises(ValueError, match=r"out must be \[T, Hq, d\]"):
        ea.attn_prefill_paged(qp, kp, kp, bt, sl, cu, 4, lse=torch.zeros(T, Hq - 1))
    with pytest.raises(ValueError, match="one value per query head"):
        ea.attn_prefill_paged(qp, kp, kp, bt, sl, cu, 4, alibi_slopes=torch.zeros(Hq + 1))

    qd = torch.zeros(S, Hq, d, dtype=bf)
    for call in (ea.attn_decode_paged, ea.attn_decode_paged_noalloc):
        with pytest.raises(ValueError, match=r"out must be \[S, Hq, d\]"):
            call(qd, kp, kp, bt, sl, out=qd[:1].contiguous())
        with pytest.raises(ValueError, match=r"out must be \[S, Hq, d\]"):
            call(qd, kp, kp, bt, sl, lse=torch.zeros(S, Hq // 2))
    k8 = kp.to(torch.int8)
    sc = torch.ones(P, Hkv)
    with pytest.raises(ValueError, match=r"out must be \[S, Hq, d\]"):
        ea.attn_decode_paged_q8(qd, k8, k8, sc, sc, bt, sl, kv_format="int8",
                                out=qd[:, :1].contiguous())
    with pytest.raises(ValueError, match="scales must be"):
        ea.attn_decode_paged_q8(qd, k8, k8, sc[:1].contiguous(), sc, bt, sl, kv_format="int8")


def test_binding_requires_one_device_per_call():
    # A kernel runs on q's device; a pointer into another device's memory is not
    # valid there, so the binding refuses such a mix (meta tensors stand in for
    # a second device here).
    import torch
    dev = torch.device("cuda", 0)
    ea._same_device(dev, k=None)
    with pytest.raises(ValueError, match="k is on meta"):
        ea._same_device(dev, k=torch.empty(2, device="meta"))
    with pytest.raises(ValueError, match="workspace is on cpu"):
        ea._same_device(dev, out=None, workspace=torch.empty(2))


def test_alignment_rules_match_the_header(lib):
    # Tensor data needs 16-byte alignment: an 8-byte-aligned q, k, v or o is refused.
    for name in ("q", "k", "v", "o"):
        assert fwd(lib, **{name: A + 8}) == INVALID, name


@pytest.mark.skipif(__import__("torch").cuda.is_available(),
                    reason="the fake addresses would reach a kernel launch on a GPU")
def test_four_byte_vectors_pass_the_alignment_check(lib):
    # A 4-byte-aligned lse (a float32 vector) passes validation; with no GPU in
    # this process the call then stops at the device lookup (ATTN_ERR_CUDA),
    # never at the argument checks.
    CUDA = 3
    assert fwd(lib, lse=A + 4) == CUDA
    assert lib.attn_fwd_ext(A, A, A, A, A + 4, 1, 2, 1, 16, 128, 0.1, 1, 0, A + 4, None) == CUDA


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    # No fallback: without the built library every entry point raises.
    missing = str(tmp_path / "libexattn.so")
    with pytest.raises(ImportError, match="not built"):
        ea.load_library(missing)
    monkeypatch.setattr(ea, "_lib", None)
    monkeypatch.setattr(ea, "LIB_PATH", missing)
    with pytest.raises(ImportError):
        ea.library()
    with pytest.raises(ImportError):
        ea.version()
    with pytest.raises(ImportError):
        ea.decode_workspace_bytes(4, 8, 128, 8)


def test_every_declaration_is_documented():
    # Each entry point in the header sits under a comment block that names it;
    # each compute entry point's block cites the passage it follows.
    text = open(os.path.join(ROOT, "include", "exattn.h")).read()
    cites = re.compile(r"Phase 08|Lab 0\d|screna|Concepts|no counterpart")
    for m in re.finditer(r"EXATTN_API[^;]*?\b(attn_[a-z0-9_]+)\s*\(", text):
        name, before = m.group(1), text[:m.start()]
        end = before.rfind("*/")
        block = before[before.rfind("/*", 0, end):end]
        assert name.replace("_workspace_bytes", "") in block or name in block, name
        assert cites.search(block), name
