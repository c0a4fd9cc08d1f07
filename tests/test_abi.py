"""Host-side checks of the C ABI (no GPU needed).

The library must load on a machine without a GPU, export every function
include/nabla.h declares, and reject bad arguments before touching the
device.
"""
import ctypes
import os
import re

import pytest

from block_sparse_attention_flatten_b200 import build as nbuild
from block_sparse_attention_flatten_b200 import nabla

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    nbuild.build()
    return nabla.lib()


def header_functions():
    text = open(os.path.join(ROOT, "include", "nabla.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(nabla_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_boundary():
    fns = header_functions()
    for name in nabla.EXPORTS:
        assert name in fns
    assert set(fns) == set(nabla.EXPORTS)


def header_prototypes():
    """name -> number of parameters, from the header's declarations."""
    text = open(os.path.join(ROOT, "include", "nabla.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    protos = {}
    for m in re.finditer(r"\b(nabla_[a-z_0-9]+)\s*\(([^)]*)\)\s*;", text):
        params = m.group(2).strip()
        protos[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return protos


def test_binding_argtypes_match_header_prototypes(lib):
    protos = header_prototypes()
    assert set(protos) == set(nabla.EXPORTS)
    for name, n in protos.items():
        assert len(getattr(lib, name).argtypes) == n, name


def test_library_exports_every_declared_symbol(lib):
    for name in header_functions():
        assert hasattr(lib, name), name


def test_strerror_covers_codes(lib):
    for code in range(0, 7):
        assert nabla.strerror(code) != "unknown error"
    assert nabla.strerror(99) == "unknown error"


def test_params_struct_layout_matches_header():
    assert ctypes.sizeof(nabla.NablaParams) == 32
    assert nabla.NablaParams.thr.offset == 4 and nabla.NablaParams.flags.offset == 24
    assert nabla.NablaParams.radial.offset == 28


def test_workspace_bytes(lib):
    prm = nabla.params(0.9)
    # pooled queries and keys (transposed), then the block-score scratch
    assert nabla.mask_workspace_bytes(1, 12, 128, 16, 48, 80, prm) == 2 * 12 * 960 * 128 * 4 + 12 * 960 * 960 * 4
    # odd block count: rows padded to a multiple of 4 columns (37 -> 40)
    assert nabla.mask_workspace_bytes(1, 1, 64, 37, 8, 8, prm) == 2 * 64 * 40 * 4 + 37 * 40 * 4
    assert nabla.mask_workspace_bytes(1, 2, 96, 4, 16, 16, prm) == 0  # D not supported
    assert nabla.mask_workspace_bytes(1, 2, 64, 4, 12, 16, prm) == 0  # H not a multiple of 8
    # key-range split: the ranges' bf16 outputs, then their fp32 LSE, each 256-byte aligned
    up = lambda x: (x + 255) // 256 * 256  # noqa: E731
    S = 64 * 48 * 80
    assert nabla.attn_split_workspace_bytes(1, 24, 128, 64, 48, 80, 4) == up(4 * S * 24 * 128 * 2) + up(4 * 24 * S * 4)
    assert nabla.attn_split_workspace_bytes(2, 3, 64, 3, 8, 24, 2) == up(2 * 2 * 576 * 3 * 64 * 2) + up(2 * 2 * 3 * 576 * 4)
    assert lib.nabla_attn_split_workspace_bytes(1, 2, 64, 4, 16, 16, 1) == 0  # nsplit < 2
    assert lib.nabla_attn_split_workspace_bytes(1, 2, 96, 4, 16, 16, 2) == 0  # D not supported


def test_invalid_arguments_rejected_before_launch(lib):
    L = lib
    s = ctypes.c_void_p(0)
    fake = ctypes.c_void_p(0x1000)
    # P must be 8; H, W multiples of P; rows a multiple of 16 bytes
    assert L.nabla_flatten(fake, ctypes.c_void_p(0x2000), 1, 4, 16, 16, 7, 128, s) == nabla.NABLA_ERR_INVALID
    assert L.nabla_flatten(fake, ctypes.c_void_p(0x2000), 1, 4, 12, 16, 8, 128, s) == nabla.NABLA_ERR_INVALID
    assert L.nabla_flatten(fake, ctypes.c_void_p(0x2000), 1, 4, 16, 16, 8, 12, s) == nabla.NABLA_ERR_INVALID
    assert L.nabla_flatten(fake, fake, 1, 4, 16, 16, 8, 128, s) == nabla.NABLA_ERR_INVALID  # aliasing
    assert L.nabla_flatten(ctypes.c_void_p(0x1001), ctypes.c_void_p(0x2000), 1, 4, 16, 16, 8, 128,
                           s) == nabla.NABLA_ERR_ALIGN
    prm = nabla.params(1.5)
    assert L.nabla_build_mask(fake, fake, 1, 2, 64, 4, 16, 16, ctypes.byref(prm), fake, fake, fake,
                              s) == nabla.NABLA_ERR_INVALID
    prm = nabla.params(0.9, sta=(2, 3, 3))
    assert L.nabla_build_mask(fake, fake, 1, 2, 64, 4, 16, 16, ctypes.byref(prm), fake, fake, fake,
                              s) == nabla.NABLA_ERR_INVALID
    prm = nabla.params(0.9)
    assert L.nabla_build_mask(fake, fake, 1, 2, 80, 4, 16, 16, ctypes.byref(prm), fake, fake, fake,
                              s) == nabla.NABLA_ERR_INVALID
    assert L.nabla_build_mask(ctypes.c_void_p(0x1008), fake, 1, 2, 64, 4, 16, 16, ctypes.byref(prm), fake, fake,
                              fake, s) == nabla.NABLA_ERR_ALIGN
    prm = nabla.params(0.9)
    a1, a2, a3 = ctypes.c_void_p(0x1000), ctypes.c_void_p(0x2000), ctypes.c_void_p(0x3000)
    assert L.nabla_flatten_pool_qk(a1, a2, a1, a3, 1, 2, 64, 4, 16, 16, ctypes.byref(prm), fake,
                                   s) == nabla.NABLA_ERR_INVALID  # q aliases qf
    assert L.nabla_flatten_pool_qk(a1, a2, a3, ctypes.c_void_p(0x4008), 1, 2, 64, 4, 16, 16, ctypes.byref(prm),
                                   fake, s) == nabla.NABLA_ERR_ALIGN
    assert L.nabla_flatten_pool_qk(a1, a2, a3, ctypes.c_void_p(0x4000), 1, 2, 96, 4, 16, 16, ctypes.byref(prm),
                                   fake, s) == nabla.NABLA_ERR_INVALID  # D
    assert L.nabla_build_mask_pooled(fake, 1, 2, 64, 4, 16, 16, ctypes.byref(prm), None, fake,
                                     s) == nabla.NABLA_ERR_INVALID
    assert L.nabla_build_mask_pooled(ctypes.c_void_p(0x1004), 1, 2, 64, 4, 16, 16, ctypes.byref(prm), fake, fake,
                                     s) == nabla.NABLA_ERR_ALIGN
    # static window: odd sizes in [1, 65535], lists present and aligned
    assert L.nabla_build_mask_sta(1, 2, 4, 16, 16, 8, 3, 2, 3, a1, a2, s) == nabla.NABLA_ERR_INVALID
    assert L.nabla_build_mask_sta(1, 2, 4, 16, 16, 8, 0, 3, 3, a1, a2, s) == nabla.NABLA_ERR_INVALID
    assert L.nabla_build_mask_sta(1, 2, 4, 16, 16, 8, 3, 3, 65537, a1, a2, s) == nabla.NABLA_ERR_INVALID
    assert L.nabla_build_mask_sta(1, 2, 4, 12, 16, 8, 3, 3, 3, a1, a2, s) == nabla.NABLA_ERR_INVALID
    assert L.nabla_build_mask_sta(1, 0, 4, 16, 16, 8, 3, 3, 3, a1, a2, s) == nabla.NABLA_ERR_INVALID
    assert L.nabla_build_mask_sta(1, 2, 4, 16, 16, 8, 3, 3, 3, None, a2, s) == nabla.NABLA_ERR_INVALID
    assert L.nabla_build_mask_sta(1, 2, 4, 16, 16, 8, 3, 3, 3, a1, ctypes.c_void_p(0x2004),
                                  s) == nabla.NABLA_ERR_ALIGN
    assert L.nabla_sparse_attn_fwd(fake, fake, fake, fake, fake, 1, 100, 2, 64, ctypes.c_float(0.0), fake, None,
                                   s) == nabla.NABLA_ERR_INVALID
    # backward: lists transposed need aligned buffers; every pointer required
    assert L.nabla_transpose_lists(a1, a2, 1, 2, 0, a3, fake, s) == nabla.NABLA_ERR_INVALID
    assert L.nabla_transpose_lists(a1, a2, 1, 2, 4, None, fake, s) == nabla.NABLA_ERR_INVALID
    assert L.nabla_transpose_lists(a1, a2, 1, 2, 4, a3, ctypes.c_void_p(0x4004), s) == nabla.NABLA_ERR_ALIGN
    p10 = [ctypes.c_void_p(0x1000 * (n + 1)) for n in range(10)]
    o4 = [ctypes.c_void_p(0x20000 + 0x1000 * n) for n in range(4)]
    f0 = ctypes.c_float(0.0)
    assert L.nabla_sparse_attn_bwd(*p10, 1, 100, 2, 64, f0, *o4, s) == nabla.NABLA_ERR_INVALID  # S % 64
    assert L.nabla_sparse_attn_bwd(*p10, 1, 128, 2, 96, f0, *o4, s) == nabla.NABLA_ERR_INVALID  # D
    assert L.nabla_sparse_attn_bwd(*p10[:5], None, *p10[6:], 1, 128, 2, 64, f0, *o4, s) == nabla.NABLA_ERR_INVALID
    assert L.nabla_sparse_attn_bwd(*p10, 1, 128, 2, 64, f0, *o4[:3], ctypes.c_void_p(0x30004),
                                   s) == nabla.NABLA_ERR_ALIGN
    assert L.nabla_sparse_attn_bwd_grid(*p10, 1, 2, 64, 2, 12, 16, f0, *o4, s) == nabla.NABLA_ERR_INVALID  # H % 8
    assert L.nabla_sparse_attn_fwd(fake, fake, fake, fake, fake, 1, 128, 2, 48, ctypes.c_float(0.0), fake, None,
                                   s) == nabla.NABLA_ERR_INVALID


def test_selftest_rejects_out_of_range_limits(lib):
    assert lib.nabla_selftest_wait_timeout(10, None) == nabla.NABLA_ERR_INVALID
    assert lib.nabla_selftest_wait_timeout(10 ** 12, None) == nabla.NABLA_ERR_INVALID


def test_binding_refuses_cpu_tensors(lib):
    import torch
    x = torch.zeros(1, 64, 8, dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        nabla.flatten(x, 1, 8, 8)


def _c_caller_source():
    """A plain C program that includes the header, takes the address of
    every declared function (so the link must resolve them all) and calls
    the host-only paths: the error strings, the workspace size arithmetic
    and an argument rejection, none of which touches a GPU."""
    fns = header_functions()
    table = ",\n    ".join(f"(void (*)(void))&{f}" for f in fns)
    return f"""#include <stdio.h>
#include <string.h>
#include "nabla.h"

static void (*const every_entry_point[])(void) = {{
    {table}
}};

int main(void) {{
  nabla_params prm;
  size_t ws;
  int rc;
  memset(&prm, 0, sizeof prm);
  prm.P = 8;
  prm.thr = 0.9f;
  ws = nabla_mask_workspace_bytes(1, 2, 64, 4, 16, 16, &prm);
  /* grid 4 x 16 x 16 = 16 blocks: pooled Q and K, fp32 [1][2][64][16]
     each, then the block scores, fp32 [1][2][16][16] */
  rc = nabla_flatten(NULL, NULL, 1, 4, 16, 16, 8, 128, NULL);
  printf("%u %zu %d %s\\n", (unsigned)(sizeof every_entry_point / sizeof every_entry_point[0]), ws, rc,
         nabla_strerror(NABLA_ERR_INVALID));
  return 0;
}}
"""


@pytest.mark.parametrize("compiler", [["gcc", "-std=c99", "-pedantic"], ["g++", "-std=c++17", "-x", "c++"]],
                         ids=["c99", "c++17"])
def test_header_compiles_links_and_rejects_from_c(lib, tmp_path, compiler):
    import subprocess
    src = tmp_path / "caller.c"
    src.write_text(_c_caller_source())
    exe = tmp_path / "caller"
    libdir = os.path.dirname(nbuild.LIB)
    cmd = compiler + ["-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                      "-L", libdir, "-lnabla", f"-Wl,-rpath,{libdir}"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split(maxsplit=3)
    assert int(out[0]) == len(header_functions())
    assert int(out[1]) == 2 * 4 * 2 * 64 * 16 + 4 * 2 * 16 * 16
    assert int(out[2]) == nabla.NABLA_ERR_INVALID  # null pointers: rejected before any CUDA call
    assert out[3].strip() == nabla.strerror(nabla.NABLA_ERR_INVALID)
