"""include/exattn.h as a C caller sees it, on the CPU.

The boundary is meant for callers in any language with a C FFI, so the header
must compile as strict C99 (and as C++), every function it declares must link
against libexattn.so, and a C program must get the same answers as the Python
binding from the calls that need no GPU: the version and status strings, the
workspace sizes, and the argument checks that run before any CUDA call.
"""
from __future__ import annotations

import os
import shutil
import subprocess

import pytest

from test_abi import ROOT, declared_functions, lib  # noqa: F401  (lib is a fixture)

import exact_io_aware_101_b200 as ea  # noqa: E402

INCLUDE = os.path.join(ROOT, "include")
LIBDIR = os.path.dirname(ea.LIB_PATH)

# A C program that names every declared function (a cast to one generic
# function-pointer type, which strict C allows) and prints what the GPU-free
# calls return.  Each compute entry point is called once with null tensors and
# must refuse them before touching the device.
C_SOURCE = r"""
#include "exattn.h"
#include <stdio.h>

typedef void (*any_fn)(void);
static const any_fn every_entry_point[] = { %(table)s };

int main(void) {
  const float scale = 0.125f;
  printf("version %%s\n", attn_version());
  for (int c = 0; c <= 4; ++c) printf("status %%d %%s\n", c, attn_status_string((attn_status_t)c));
  printf("decode_ws %%zu %%zu\n", attn_decode_workspace_bytes(4, 8, 128, 8, 16),
         attn_decode_workspace_bytes(64, 32, 128, 512, 16));
  printf("bwd_ws %%zu\n", attn_bwd_workspace_bytes(2, 16, 1000));
  printf("fwd %%d\n", (int)attn_fwd(NULL, NULL, NULL, NULL, NULL, 1, 1, 1, 8, 64, scale, 0, NULL));
  printf("fwd_f32 %%d\n",
         (int)attn_fwd_f32(NULL, NULL, NULL, NULL, NULL, 1, 1, 1, 8, 64, scale, 0, NULL));
  printf("decode %%d\n", (int)attn_decode_paged(NULL, NULL, NULL, NULL, NULL, NULL, NULL, 4, 8, 2,
                                                128, 16, 8, 100, scale, NULL, 0, NULL));
  printf("noalloc %%d\n", (int)attn_decode_paged_noalloc(NULL, NULL, NULL, NULL, NULL, NULL, NULL,
                                                         4, 8, 2, 128, 16, 8, 100, scale, NULL));
  printf("bwd %%d\n", (int)attn_bwd(NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 1, 1, 1,
                                    8, 64, scale, 0, 0, NULL, NULL, 0, NULL));
  {
    unsigned st = 7u;
    printf("read_status %%d %%u\n", (int)attn_decode_read_status(NULL, &st), st);
  }
  printf("entry_points %%d\n", (int)(sizeof every_entry_point / sizeof every_entry_point[0]));
  return 0;
}
"""


def _c_program(tmp_path):
    names = sorted(declared_functions())
    src = C_SOURCE % {"table": ", ".join("(any_fn)%s" % n for n in names)}
    path = tmp_path / "caller.c"
    path.write_text(src)
    return path, names


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_header_is_strict_c99_and_links(tmp_path, lib):  # noqa: F811
    src, names = _c_program(tmp_path)
    exe = tmp_path / "caller"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", INCLUDE, str(src), "-L", LIBDIR, "-lexattn",
                    "-Wl,-rpath," + LIBDIR, "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    got = dict(line.split(" ", 1) for line in out.strip().splitlines() if not
               line.startswith("status "))
    statuses = [line.split(" ", 2)[1:] for line in out.splitlines() if line.startswith("status ")]

    assert got["version"] == ea.version()
    assert statuses == [[str(c), ea.status_string(c)] for c in range(5)]
    assert got["decode_ws"] == "%d %d" % (lib.attn_decode_workspace_bytes(4, 8, 128, 8, 16),
                                          lib.attn_decode_workspace_bytes(64, 32, 128, 512, 16))
    assert got["bwd_ws"] == str(ea.bwd_workspace_bytes(2, 16, 1000))
    for call in ("fwd", "fwd_f32", "decode", "noalloc", "bwd"):
        assert got[call] == "1", call  # ATTN_ERR_INVALID_ARG, before any CUDA call
    assert got["read_status"] == "1 7"  # refused, and nothing written
    assert got["entry_points"] == str(len(names))


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_header_compiles_as_cpp(tmp_path):
    src = tmp_path / "caller.cpp"
    src.write_text('#include "exattn.h"\n'
                   'static_assert(sizeof(attn_status_t) == sizeof(int), "enum is int-sized");\n'
                   'int main() { return attn_status_string(ATTN_OK)[0] == \'A\' ? 0 : 1; }\n')
    subprocess.run(["g++", "-std=c++17", "-Wall", "-Wextra", "-Werror", "-I", INCLUDE,
                    "-fsyntax-only", str(src)], check=True)
