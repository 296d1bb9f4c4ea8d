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
