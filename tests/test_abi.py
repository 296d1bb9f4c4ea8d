"""The C-ABI library builds, loads and exports every entry point include/nvfp4moe.h
declares; host-only calls work without a GPU (CPU only: no kernel is launched)."""
import ctypes
import subprocess

import pytest

import nvfp4_quantized_moe_group_b200 as moe
from nvfp4_quantized_moe_group_b200 import build as build_mod


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return moe.lib()


def test_every_declared_symbol_is_exported(lib):
    declared = moe.declared_symbols()
    assert len(declared) >= 16
    out = subprocess.run(["nm", "-D", "--defined-only", moe.LIB_PATH], capture_output=True, text=True, check=True)
    exported = {line.split()[-1] for line in out.stdout.splitlines() if "nvfp4moe_" in line}
    assert set(declared) == exported
    for name in declared:
        assert getattr(lib, name) is not None


def test_host_only_calls(lib):
    c = moe.cfg_default()
    assert (c.E, c.n_groups, c.topk_groups, c.topk, c.H, c.I) == (256, 8, 4, 8, 5120, 2560)
    assert abs(c.routed_scale - 2.5) == 0
    assert lib.nvfp4moe_cfg_check(ctypes.byref(c)) == moe.OK
    bad = moe.Cfg(256, 8, 4, 8, 5000, 2560, 2.5)
    assert lib.nvfp4moe_cfg_check(ctypes.byref(bad)) == moe.ERR_SHAPE
    bad = moe.Cfg(256, 8, 9, 8, 5120, 2560, 2.5)
    assert lib.nvfp4moe_cfg_check(ctypes.byref(bad)) == moe.ERR_SHAPE
    assert moe.forward_workspace_bytes(c, 4096) > 4096 * 5120 * 4
    assert moe.forward_workspace_bytes(c, 0) == 0
    assert moe.route_workspace_bytes(c, 16) > 0
    assert moe.swizzled_scale_bytes(129, 6) == 256 * 8
    assert moe.quantize_workspace_bytes(10, 64) >= 256
    assert moe.status_string(moe.ERR_TIMEOUT) == "bounded device wait ran out"


def test_argument_errors_return_without_gpu(lib):
    # shape and pointer checks happen before any device call
    assert lib.nvfp4moe_quantize(None, 4, 63, None, None, None, 0, None, None, 0, None) == moe.ERR_SHAPE
    assert lib.nvfp4moe_quantize(None, 4, 64, None, None, None, 7, None, None, 0, None) == moe.ERR_ARG
    c = moe.cfg_default()
    assert lib.nvfp4moe_route(ctypes.byref(c), None, 4, None, None, None, None, None, 0, None) == moe.ERR_ARG
    assert lib.nvfp4moe_forward(None, None, 4, None, None, None, None, None, 0, None) == moe.ERR_ARG


C_PROGRAM = r"""
#include <stdio.h>
#include "nvfp4moe.h"
int main(void) {
  nvfp4moe_cfg c;
  if (nvfp4moe_cfg_default(&c) != NVFP4MOE_OK) return 1;
  if (nvfp4moe_cfg_check(&c) != NVFP4MOE_OK) return 2;
  size_t ws = nvfp4moe_workspace_bytes(&c, 16);
  if (ws == 0 || ws != nvfp4moe_forward_workspace_bytes(&c, 16)) return 3;
  if (nvfp4moe_quantize(NULL, 4, 63, NULL, NULL, NULL, 0, NULL, NULL, 0, NULL) != NVFP4MOE_ERR_SHAPE) return 4;
  printf("%d %d %d %d %d %d %s\n", c.E, c.n_groups, c.topk_groups, c.topk, c.H, c.I,
         nvfp4moe_status_string(NVFP4MOE_ERR_SHAPE));
  return 0;
}
"""


def test_header_is_plain_c_and_links_from_c(lib):
    """include/nvfp4moe.h compiles as C99 and C++17, and a C program links against the library
    and calls its host-only entry points (built under the git-ignored _build/)."""
    import os
    import pathlib
    root = os.path.dirname(os.path.dirname(moe.LIB_PATH))
    inc = os.path.join(root, "include")
    tmp_path = pathlib.Path(root, "_build", "abi_c")
    tmp_path.mkdir(parents=True, exist_ok=True)
    hdr = os.path.join(inc, "nvfp4moe.h")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-fsyntax-only", "-x", "c", hdr],
                   check=True)
    subprocess.run(["g++", "-std=c++17", "-Wall", "-Werror", "-fsyntax-only", "-x", "c++", hdr], check=True)
    src = tmp_path / "main.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "main"
    libdir = os.path.dirname(moe.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", inc, str(src), "-L", libdir, "-lnvfp4moe",
                    f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out
    assert out.stdout.split()[:6] == ["256", "8", "4", "8", "5120", "2560"]
    assert "unsupported shape" in out.stdout
