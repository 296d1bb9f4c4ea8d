"""nvfp4moe_route_noalloc: the router for callers that cannot allocate device memory.

Such callers (a host runtime that hands the library only input and output buffers and
forbids device allocation after start-up, or a host framework that owns all device memory)
cannot provide the workspace nvfp4moe_route needs, so this entry point keeps the router's
scratch in a fixed device array of the library.  These tests call it through the C ABI on
consecutive calls (the array keeps the previous call's contents) and judge every call
against the oracle's routing under the near-tie protocol, with the error bound of the FP32
logits this call computes; against nvfp4moe_route (whose logits for T > 64 come from the
integer tensor-core path, with a tighter bound) they require equal selections on every
token that is clean under the FP32 bound, since only there are both selections fixed.  A call
beyond the array's capacity must be refused.  The file is collected last so that a failure
here does not hide the other GPU tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import nvfp4_quantized_moe_group_b200 as moe
from workloads import TINY, BEAM, activations, router_weight, zipf_bias
from tests.helpers import cfg_ns, check_routing, router_logit_bound_fp32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    moe.lib()


def _route_noalloc(cfg, x, wr, bias, idx, w):
    f = moe.lib().nvfp4moe_route_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.POINTER(moe.Cfg), ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    ptr = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())  # noqa: E731
    return f(ctypes.byref(cfg), ptr(x), x.shape[0], ptr(wr), ptr(bias), ptr(idx), ptr(w),
             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _cfg(shape):
    return moe.make_cfg(shape.E, shape.n_groups, shape.topk_groups, shape.topk, shape.H, shape.I,
                        shape.routed_scale)


def _judge(shape, x, wr, bias, idx, w):
    """The call's selection and weights against the oracle (near-tie protocol, FP32 bound);
    returns the mask of tokens clean under that bound."""
    xn = x.float().cpu().numpy().astype(np.float64)
    wn = wr.cpu().numpy().astype(np.float64)
    bn = None if bias is None else bias.cpu().numpy().astype(np.float64)
    r = oracle.route(xn, wn, cfg_ns(shape), bn)
    clean, _ = check_routing(idx.cpu().numpy(), w.cpu().numpy(), r, xn, wn, bn, shape,
                             bound=router_logit_bound_fp32)
    return clean


@pytest.mark.parametrize("order", [0, 1])
def test_matches_oracle_and_route_on_consecutive_calls(order):
    cases = [(BEAM, 4096, False, None), (BEAM, 16, True, None), (TINY, 64, False, None),
             (BEAM, 1000, False, zipf_bias(256))]
    if order:
        cases = cases[::-1]
    for shape, T, rms, bias in cases:
        cfg = _cfg(shape)
        x = activations(T, shape, rms_rows=rms).cuda()
        wr = router_weight(shape).cuda()
        b = None if bias is None else bias.cuda()
        idx = torch.full((T, shape.topk), -1, dtype=torch.int32, device="cuda")
        w = torch.full((T, shape.topk), -1.0, dtype=torch.float32, device="cuda")
        assert _route_noalloc(cfg, x, wr, b, idx, w) == moe.OK
        ref_idx, ref_w = moe.route(cfg, x, wr, b)
        torch.cuda.synchronize()
        assert moe.last_device_status() == moe.OK
        clean = _judge(shape, x, wr, bias, idx, w)
        assert clean.mean() > 0.9
        got, ref = idx.cpu().numpy(), ref_idx.cpu().numpy()
        np.testing.assert_array_equal(got[clean], ref[clean])
        np.testing.assert_allclose(w.cpu().numpy()[clean], ref_w.cpu().numpy()[clean], rtol=2e-6, atol=0)


def test_refuses_calls_beyond_capacity():
    cfg = _cfg(BEAM)
    wr = router_weight(BEAM).cuda()
    x = activations(4737, BEAM).cuda()
    idx = torch.empty((4737, 8), dtype=torch.int32, device="cuda")
    w = torch.empty((4737, 8), dtype=torch.float32, device="cuda")
    assert _route_noalloc(cfg, x, wr, None, idx, w) == moe.ERR_WORKSPACE
    x = x[:4736].contiguous()
    assert _route_noalloc(cfg, x, wr, None, idx[:4736], w[:4736]) == moe.OK
    torch.cuda.synchronize()
    assert moe.last_device_status() == moe.OK
    _judge(BEAM, x, wr, None, idx[:4736], w[:4736])


def test_status_of_the_fixed_scratch():
    """The call's device status (here a NaN router row) is read through
    nvfp4moe_last_device_status, the one reader of the fixed scratch's status word; the
    selection still holds topk distinct in-range experts, the NaN expert ranked last."""
    cfg = _cfg(BEAM)
    x = activations(16, BEAM, seed=5).cuda()
    wr = router_weight(BEAM).cuda()
    idx = torch.empty((16, 8), dtype=torch.int32, device="cuda")
    w = torch.empty((16, 8), dtype=torch.float32, device="cuda")
    assert _route_noalloc(cfg, x, wr, None, idx, w) == moe.OK
    assert moe.last_device_status() == moe.OK
    wr[3, 7] = float("nan")
    assert _route_noalloc(cfg, x, wr, None, idx, w) == moe.OK
    assert moe.last_device_status() == moe.ERR_NONFINITE
    got = idx.cpu().numpy()
    assert ((got >= 0) & (got < BEAM.E)).all() and not (got == 3).any()
    assert all(len(set(row.tolist())) == 8 for row in got)
