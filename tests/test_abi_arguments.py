"""Argument checking of every C-ABI entry point, on a machine without a GPU.

include/nvfp4moe.h documents, per call, the shapes and pointers it accepts and the status it
returns otherwise.  Every check below happens on the host before any CUDA call, so these
calls return their documented status here; a call that passes every host check reaches the
device check and fails with NVFP4MOE_ERR_DEVICE or NVFP4MOE_ERR_CUDA (the library has no CPU
path).  The pointers passed are placeholders that are never dereferenced: the library reads
no device pointer on the host.  The module is skipped where a GPU is present, since there a
call that passed its checks would launch kernels on the placeholders.
"""
import ctypes

import pytest
import torch

import nvfp4_quantized_moe_group_b200 as moe
from nvfp4_quantized_moe_group_b200 import build as build_mod
from nvfp4_quantized_moe_group_b200._lib import ExpertTensors

pytestmark = pytest.mark.skipif(torch.cuda.is_available(),
                                reason="placeholder device pointers: host-only checks, no GPU")

A = 1 << 20                       # a 16-byte (and 256-byte) aligned placeholder address
MIS = A + 8                       # 8-byte aligned, not 16
BIG = 1 << 40
NO_DEVICE = (moe.ERR_DEVICE, moe.ERR_CUDA)


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return moe.lib()


def _cfg(**kw):
    c = moe.cfg_default()
    for k, v in kw.items():
        setattr(c, k, v)
    return c


@pytest.mark.parametrize("field,value,want", [
    ("H", 5000, "SHAPE"), ("H", 0, "SHAPE"), ("I", 2500, "SHAPE"), ("I", -128, "SHAPE"),
    ("E", 0, "SHAPE"), ("E", 257, "SHAPE"), ("n_groups", 0, "SHAPE"), ("n_groups", 3, "SHAPE"),
    ("n_groups", 4, "SHAPE"),         # 64 experts per group: above the 32 a group may hold
    ("topk_groups", 0, "SHAPE"), ("topk_groups", 9, "SHAPE"),
    ("topk", 0, "SHAPE"), ("topk", 9, "SHAPE"),
    ("routed_scale", float("nan"), "ARG"),
])
def test_cfg_limits(lib, field, value, want):
    c = _cfg(**{field: value})
    assert lib.nvfp4moe_cfg_check(ctypes.byref(c)) == getattr(moe, f"ERR_{want}")
    assert lib.nvfp4moe_forward_workspace_bytes(ctypes.byref(c), 16) == 0
    assert lib.nvfp4moe_route_workspace_bytes(ctypes.byref(c), 16) == 0


def test_cfg_small_layers_accepted(lib):
    for kw in ({"E": 8, "n_groups": 1, "topk_groups": 1, "topk": 1},
               {"E": 32, "n_groups": 8, "topk_groups": 4, "topk": 8, "H": 256, "I": 128}):
        c = _cfg(**kw)
        assert lib.nvfp4moe_cfg_check(ctypes.byref(c)) == moe.OK
    c = _cfg(E=8, n_groups=4, topk_groups=1, topk=3)      # 3 experts from one group of 2
    assert lib.nvfp4moe_cfg_check(ctypes.byref(c)) == moe.ERR_SHAPE
    assert lib.nvfp4moe_cfg_check(None) == moe.ERR_ARG
    assert lib.nvfp4moe_cfg_default(None) == moe.ERR_ARG


def test_quantize_checks(lib):
    q = lib.nvfp4moe_quantize
    ws_n = moe.quantize_workspace_bytes(4, 64)
    ok = dict(x=A, rows=4, cols=64, g_in=None, codes=A, scales=A, layout=0, g_out=None, ws=A, ws_n=ws_n)

    def call(**kw):
        a = {**ok, **kw}
        return q(a["x"], a["rows"], a["cols"], a["g_in"], a["codes"], a["scales"], a["layout"], a["g_out"],
                 a["ws"], a["ws_n"], None)

    assert call(cols=63) == moe.ERR_SHAPE
    assert call(cols=0) == moe.ERR_SHAPE
    assert call(cols=1 << 31) == moe.ERR_SHAPE
    assert call(rows=-1) == moe.ERR_SHAPE
    assert call(rows=(1 << 31) - 128) == moe.ERR_SHAPE
    assert call(rows=1 << 20, cols=1 << 20) == moe.ERR_SHAPE          # rows * cols = 2^40
    assert call(rows=1 << 62, cols=1 << 30) == moe.ERR_SHAPE          # no overflow of rows * cols
    assert call(layout=7) == moe.ERR_ARG
    assert call(ws=None) == moe.ERR_ARG
    assert call(ws=MIS) == moe.ERR_ARG
    assert call(scales=None) == moe.ERR_ARG
    assert call(scales=A + 2) == moe.ERR_ARG
    assert call(x=None) == moe.ERR_ARG
    assert call(x=MIS) == moe.ERR_ARG
    assert call(codes=MIS) == moe.ERR_ARG
    assert call(ws_n=ws_n - 1) == moe.ERR_WORKSPACE
    assert call() in NO_DEVICE
    assert call(rows=0, x=None, codes=None, scales=None) in NO_DEVICE   # empty input: pointers unused


def test_quantize_weights_lh_checks(lib):
    f = lib.nvfp4moe_quantize_weights_lh
    ws_n = moe.quantize_workspace_bytes(4, 64)
    ok = dict(w=A, rows=4, cols=64, h=A, m=4, codes=A, scales=A, g=A, ws=A, ws_n=ws_n)

    def call(**kw):
        a = {**ok, **kw}
        return f(a["w"], a["rows"], a["cols"], a["h"], a["m"], a["codes"], a["scales"], a["g"], a["ws"],
                 a["ws_n"], None)

    assert call(rows=0) == moe.ERR_SHAPE
    assert call(cols=8) == moe.ERR_SHAPE
    assert call(cols=16 * 65536) == moe.ERR_SHAPE
    assert call(rows=1 << 31) == moe.ERR_SHAPE
    assert call(rows=1 << 62) == moe.ERR_SHAPE
    assert call(m=-1) == moe.ERR_ARG
    assert call(m=17) == moe.ERR_ARG
    for k in ("w", "h", "codes", "scales", "g", "ws"):
        assert call(**{k: None}) == moe.ERR_ARG, k
    assert call(w=MIS) == moe.ERR_ARG
    assert call(ws_n=ws_n - 1) == moe.ERR_WORKSPACE
    assert call() in NO_DEVICE


def test_route_checks(lib):
    c = moe.cfg_default()
    ws_n = moe.route_workspace_bytes(c, 16)
    r = lib.nvfp4moe_route

    def call(cfg=c, x=A, T=16, w=A, idx=A, wts=A, ws=A, n=ws_n):
        return r(ctypes.byref(cfg) if cfg is not None else None, x, T, w, None, idx, wts, ws, n, None)

    assert call(cfg=None) == moe.ERR_ARG
    assert call(cfg=_cfg(H=100)) == moe.ERR_SHAPE
    assert call(T=-1) == moe.ERR_SHAPE
    assert call(T=(1 << 24) + 1) == moe.ERR_SHAPE
    assert call(ws=None) == moe.ERR_ARG
    for k in ("x", "w", "idx", "wts"):
        assert call(**{k: None}) == moe.ERR_ARG, k
    assert call(x=MIS) == moe.ERR_ARG
    assert call(n=ws_n - 1) == moe.ERR_WORKSPACE
    assert call() in NO_DEVICE
    assert call(T=0, x=None, w=None, idx=None, wts=None) in NO_DEVICE


def test_expert_handles_checks(lib):
    c = moe.cfg_default()
    h = ctypes.c_void_p()
    assert lib.nvfp4moe_experts_create(ctypes.byref(c), None) == moe.ERR_ARG
    assert lib.nvfp4moe_experts_create(ctypes.byref(_cfg(topk=0)), ctypes.byref(h)) == moe.ERR_SHAPE
    assert h.value is None
    for b, n in ((-1, 4), (0, 0), (250, 7), (256, 1)):
        assert lib.nvfp4moe_experts_create_local(ctypes.byref(c), b, n, ctypes.byref(h)) == moe.ERR_ARG, (b, n)
    assert lib.nvfp4moe_experts_create(ctypes.byref(c), ctypes.byref(h)) in NO_DEVICE
    assert h.value is None
    assert lib.nvfp4moe_fp8_experts_create(ctypes.byref(c), None) == moe.ERR_ARG
    assert lib.nvfp4moe_fp8_experts_create(ctypes.byref(c), ctypes.byref(h)) in NO_DEVICE
    t = ExpertTensors()
    assert lib.nvfp4moe_experts_set(None, 0, ctypes.byref(t), None) == moe.ERR_ARG
    assert lib.nvfp4moe_fp8_experts_set(None, 0, None, None) == moe.ERR_ARG
    lo, n = ctypes.c_int32(), ctypes.c_int32()
    assert lib.nvfp4moe_experts_range(None, ctypes.byref(lo), ctypes.byref(n)) == moe.ERR_ARG
    assert lib.nvfp4moe_experts_cfg(None, ctypes.byref(c)) == moe.ERR_ARG
    lib.nvfp4moe_experts_destroy(None)
    lib.nvfp4moe_fp8_experts_destroy(None)


def test_forward_family_without_a_handle(lib):
    for name in ("nvfp4moe_forward", "nvfp4moe_forward_partial", "nvfp4moe_forward_fp8"):
        assert getattr(lib, name)(None, A, 16, A, None, A, None, A, 1 << 30, None) == moe.ERR_ARG, name
    assert lib.nvfp4moe_forward_residual(None, A, 16, A, 1e-6, 2, A, None, A, None, A, 1 << 30, None) == moe.ERR_ARG


def test_finalize_checks(lib):
    f = lib.nvfp4moe_finalize
    assert f(A, 7, A, None) == moe.ERR_SHAPE
    assert f(A, -8, A, None) == moe.ERR_SHAPE
    assert f(A, BIG, A, None) == moe.ERR_SHAPE
    assert f(None, 0, None, None) == moe.OK                          # nothing to do, no device call
    assert f(None, 8, A, None) == moe.ERR_ARG
    assert f(A, 8, MIS, None) == moe.ERR_ARG
    assert f(A, 8, A, None) in NO_DEVICE


def test_quantize_fp8_checks(lib):
    f = lib.nvfp4moe_quantize_fp8
    ws_n = moe.quantize_workspace_bytes(4, 64)

    def call(x=A, rows=4, cols=64, codes=A, scales=A, ws=A, n=ws_n):
        return f(x, rows, cols, codes, scales, ws, n, None)

    assert call(rows=0) == moe.ERR_SHAPE
    assert call(cols=8) == moe.ERR_SHAPE
    assert call(cols=1 << 31) == moe.ERR_SHAPE
    assert call(rows=1 << 31) == moe.ERR_SHAPE
    assert call(rows=1 << 62, cols=1 << 30) == moe.ERR_SHAPE
    assert call(rows=1 << 24, cols=1 << 16) == moe.ERR_SHAPE          # rows * cols = 2^40
    for k in ("x", "codes", "scales", "ws"):
        assert call(**{k: None}) == moe.ERR_ARG, k
    assert call(codes=A + 4) == moe.ERR_ARG
    assert call(n=ws_n - 1) == moe.ERR_WORKSPACE
    assert call() in NO_DEVICE


def test_status_calls(lib):
    assert lib.nvfp4moe_status_read(None, None) == moe.ERR_ARG
    for code in (moe.OK, moe.ERR_ARG, moe.ERR_SHAPE, moe.ERR_CUDA, moe.ERR_WORKSPACE, moe.ERR_NONFINITE,
                 moe.ERR_TIMEOUT, moe.ERR_DEVICE):
        assert moe.status_string(code) != "unknown status"
    assert moe.status_string(12345) == "unknown status"


def test_route_noalloc_checks(lib):
    c = moe.cfg_default()
    r = lib.nvfp4moe_route_noalloc

    def call(cfg=c, x=A, T=16, w=A, idx=A, wts=A):
        return r(ctypes.byref(cfg) if cfg is not None else None, x, T, w, None, idx, wts, None)

    assert call(cfg=None) == moe.ERR_ARG
    assert call(cfg=_cfg(topk=9)) == moe.ERR_SHAPE
    assert call(T=-1) == moe.ERR_SHAPE
    assert call(T=(1 << 24) + 1) == moe.ERR_SHAPE
    for k in ("x", "w", "idx", "wts"):
        assert call(**{k: None}) == moe.ERR_ARG, k
    assert call(w=MIS) == moe.ERR_ARG
    assert call(T=4737) == moe.ERR_WORKSPACE                   # T * E above the fixed scratch
    assert call(T=4736) in NO_DEVICE


def test_failed_calls_report_no_launches(lib):
    """A call rejected on the host enqueued nothing, and the launch count says so."""
    c = moe.cfg_default()
    calls = [
        lambda: lib.nvfp4moe_quantize(None, 4, 63, None, None, None, 0, None, None, 0, None),
        lambda: lib.nvfp4moe_route(ctypes.byref(c), None, -1, None, None, None, None, None, 0, None),
        lambda: lib.nvfp4moe_forward(None, A, 16, A, None, A, None, A, 1 << 30, None),
        lambda: lib.nvfp4moe_forward_partial(None, A, 16, A, None, None, None, A, 1 << 30, None),
        lambda: lib.nvfp4moe_finalize(A, 7, A, None),
        lambda: lib.nvfp4moe_quantize_fp8(None, 0, 16, None, None, None, 0, None),
    ]
    for f in calls:
        assert f() != moe.OK
        assert lib.nvfp4moe_last_launch_count() == 0


def test_status_and_workspace_aliases(lib):
    # no call on this thread has reached the device, so no status word has been recorded
    assert lib.nvfp4moe_last_device_status(None) == moe.ERR_ARG
    c = moe.cfg_default()
    for T in (1, 16, 4096):
        assert lib.nvfp4moe_workspace_bytes(ctypes.byref(c), T) == moe.forward_workspace_bytes(c, T) > 0
    assert lib.nvfp4moe_workspace_bytes(ctypes.byref(c), 0) == 0
    assert lib.nvfp4moe_workspace_bytes(ctypes.byref(_cfg(H=100)), 16) == 0


def test_expert_parallel_exchange_checks(lib):
    """nvfp4moe_amax, _ep_dispatch, _ep_experts and _ep_combine: the documented host-side checks."""
    c = moe.cfg_default()
    ws_q = moe.quantize_workspace_bytes(16, 5120)
    assert lib.nvfp4moe_amax(A, 16, 5120, None, A, ws_q, None) == moe.ERR_ARG
    assert lib.nvfp4moe_amax(A, 16, 5121, A, A, ws_q, None) == moe.ERR_SHAPE
    assert lib.nvfp4moe_amax(MIS, 16, 5120, A, A, ws_q, None) == moe.ERR_ARG
    assert lib.nvfp4moe_amax(A, 16, 5120, A, A, 8, None) == moe.ERR_WORKSPACE
    assert lib.nvfp4moe_amax(A, 16, 5120, A, A, ws_q, None) in NO_DEVICE

    wsd = moe.ep_dispatch_workspace_bytes(c, 16)
    assert wsd > 0 and moe.ep_dispatch_workspace_bytes(_cfg(H=100), 16) == 0

    def dispatch(cfg=c, G=8, x=A, T=16, w=A, amax=A, codes=A, scales=A, ws_bytes=wsd):
        return lib.nvfp4moe_ep_dispatch(ctypes.byref(cfg), G, x, T, w, None, amax, codes, scales, A, A, A, A, A,
                                        ws_bytes, None)

    assert dispatch(G=3) == moe.ERR_ARG                 # 256 experts do not split over 3 ranks
    assert dispatch(G=0) == moe.ERR_ARG
    assert dispatch(T=0) == moe.ERR_SHAPE
    for k in ("x", "w", "amax", "codes", "scales"):
        assert dispatch(**{k: None}) == moe.ERR_ARG, k
    assert dispatch(codes=MIS) == moe.ERR_ARG
    assert dispatch(ws_bytes=wsd - 1) == moe.ERR_WORKSPACE
    assert dispatch() in NO_DEVICE

    assert moe.ep_experts_workspace_bytes(c, 32, 4096) > 0
    assert moe.ep_experts_workspace_bytes(c, 0, 4096) == 0
    assert moe.ep_experts_workspace_bytes(c, 257, 4096) == 0
    assert lib.nvfp4moe_ep_experts(None, A, A, A, A, 16, A, A, A, 1 << 30, None) == moe.ERR_ARG

    assert lib.nvfp4moe_ep_combine(A, A, 16, 9, 5120, A, None) == moe.ERR_SHAPE
    assert lib.nvfp4moe_ep_combine(A, A, 16, 8, 5000, A, None) == moe.ERR_SHAPE
    assert lib.nvfp4moe_ep_combine(None, A, 16, 8, 5120, A, None) == moe.ERR_ARG
    assert lib.nvfp4moe_ep_combine(MIS, A, 16, 8, 5120, A, None) == moe.ERR_ARG
    assert lib.nvfp4moe_ep_combine(A, A, 0, 8, 5120, A, None) == moe.OK
    assert lib.nvfp4moe_ep_combine(A, A, 16, 8, 5120, A, None) in NO_DEVICE


def test_peer_combine_checks(lib):
    """nvfp4moe_forward_partial_peer and the inter-process handle calls: host-side checks."""
    f = lib.nvfp4moe_forward_partial_peer

    def call(x=None, T=16, peers=A, n=2, rows=8, dbg=None):
        return f(x, A, T, A, None, peers, n, rows, dbg, A, 1 << 30, None)

    assert call(peers=None) == moe.ERR_ARG
    assert call(peers=A + 4) == moe.ERR_ARG                     # the pointer table is 8-byte aligned
    assert call(n=0) == moe.ERR_SHAPE
    assert call(rows=0) == moe.ERR_SHAPE
    assert call(n=3, rows=5) == moe.ERR_SHAPE                   # n_peers * rows_per_peer != T
    d = moe._lib.Debug()
    d.acc = A                                                   # the sums live in the peers
    assert call(dbg=ctypes.byref(d)) == moe.ERR_ARG
    assert call() == moe.ERR_ARG                                # no expert handle
    assert lib.nvfp4moe_last_launch_count() == 0
    buf = ctypes.create_string_buffer(64)
    off = ctypes.c_int64()
    assert lib.nvfp4moe_ipc_get_handle(None, buf, ctypes.byref(off)) == moe.ERR_ARG
    assert lib.nvfp4moe_ipc_get_handle(A, None, ctypes.byref(off)) == moe.ERR_ARG
    assert lib.nvfp4moe_ipc_get_handle(A, buf, None) == moe.ERR_ARG
    assert lib.nvfp4moe_ipc_get_handle(A, buf, ctypes.byref(off)) in NO_DEVICE
    p = ctypes.c_void_p()
    assert lib.nvfp4moe_ipc_open(None, ctypes.byref(p)) == moe.ERR_ARG
    assert lib.nvfp4moe_ipc_open(buf, None) == moe.ERR_ARG
    assert lib.nvfp4moe_ipc_open(buf, ctypes.byref(p)) in NO_DEVICE
    assert lib.nvfp4moe_ipc_close(None) == moe.ERR_ARG
    assert lib.nvfp4moe_ipc_close(A) in NO_DEVICE
