"""Failure detection on the GPU without a GPU fault.

Every wait of the layer's kernels on another CTA or on the tensor cores is bounded.  These
tests make one run out on purpose, through the call's own test hook (one CTA of the fused
front-end kernel skips its arrival at the first grid barrier, with a 5 ms wait limit), and
check what a caller sees: NVFP4MOE_ERR_TIMEOUT in the status word after about the limit, no
work done by the later kernels of the call (the accumulator, zeroed before the barrier,
reaches the output as zeros), and a usable context whose next clean call gives the clean
result.  A short wait limit on a normal call must not raise a timeout.  A workspace filled
with 0xFF bytes before the call must give the same results as a zeroed one: no kernel reads
workspace memory the call has not written.
"""
import time

import numpy as np
import pytest
import torch

import nvfp4_quantized_moe_group_b200 as moe
from workloads import TINY, BEAM, activations, router_weight
from tests.helpers import bf16_half_ulp
from tests.test_gpu_forward import gpu_experts

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    moe.lib()


def _within_one_bf16_unit(a: torch.Tensor, b: torch.Tensor) -> bool:
    """The 8 weighted expert rows of a token are added with FP32 atomics in no fixed order, so
    two clean calls agree to one BF16 unit in the last place, except where the rows cancel:
    there the FP32 sums differ by a few units of 2^-24 of the rows' own magnitude, which can
    exceed a BF16 unit of the small result (bounded here by 2^-16 of the token row's largest
    output)."""
    a, b = a.float().cpu().numpy(), b.float().cpu().numpy()
    row = np.abs(b).max(axis=1, keepdims=True)
    return bool(np.all(np.abs(a - b) <= 2 * bf16_half_ulp(b) + 2.0 ** -16 * row + 1e-30))


@pytest.mark.parametrize("shape,cta", [(TINY, 1), (BEAM, 1), (BEAM, 2)])
def test_front_barrier_timeout_is_reported_and_contained(shape, cta):
    ex = gpu_experts(shape)
    T = 16
    x = activations(T, shape, seed=31).cuda()
    wr = router_weight(shape).cuda()
    ws = torch.empty(moe.forward_workspace_bytes(ex.cfg, T), dtype=torch.uint8, device="cuda")
    ref = moe.forward(ex, x, wr, ws=ws).clone()
    assert moe.status_read(ws) == moe.OK
    out = torch.full_like(ref, float("nan"))
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    moe.forward(ex, x, wr, out=out, ws=ws, wait_limit_us=5000, inject_skip_arrive=cta)
    st = moe.status_read(ws)
    elapsed = time.perf_counter() - t0
    assert st == moe.ERR_TIMEOUT
    assert elapsed < 1.0, f"the call took {elapsed:.2f} s: the 5 ms limit was not applied"
    assert bool((out == 0).all()), "the GEMMs after the timed-out front end must do no work"
    # the context is usable and the next clean call on the same workspace is clean
    again = moe.forward(ex, x, wr, ws=ws)
    assert moe.status_read(ws) == moe.OK
    assert _within_one_bf16_unit(again, ref)
    assert moe.last_device_status() == moe.OK


def test_test_hook_needs_the_fused_front_end():
    """The hook exists only in the fused front end (T <= 64): a larger call that asks for it is
    refused on the host and enqueues nothing."""
    ex = gpu_experts(TINY)
    T = 130
    x = activations(T, TINY, seed=32).cuda()
    wr = router_weight(TINY).cuda()
    with pytest.raises(moe.NvFp4MoeError) as e:
        moe.forward(ex, x, wr, inject_skip_arrive=1)
    assert e.value.status == moe.ERR_ARG
    assert moe.last_launch_count() == 0
    with pytest.raises(moe.NvFp4MoeError):
        moe.forward(ex, x[:16].contiguous(), wr, inject_skip_arrive=-1)


@pytest.mark.parametrize("shape,T", [(TINY, 16), (TINY, 130), (BEAM, 16), (BEAM, 1100)])
def test_short_wait_limit_on_a_normal_call(shape, T):
    """A 200 ms limit is far above every wait of a normal call: no timeout, same result."""
    ex = gpu_experts(shape)
    x = activations(T, shape, seed=33).cuda()
    wr = router_weight(shape).cuda()
    ws = torch.empty(moe.forward_workspace_bytes(ex.cfg, T), dtype=torch.uint8, device="cuda")
    ref = moe.forward(ex, x, wr, ws=ws).clone()
    assert moe.status_read(ws) == moe.OK
    got = moe.forward(ex, x, wr, ws=ws, wait_limit_us=200_000)
    assert moe.status_read(ws) == moe.OK
    assert _within_one_bf16_unit(got, ref)


@pytest.mark.parametrize("shape,T", [(TINY, 16), (TINY, 130), (BEAM, 16), (BEAM, 1100)])
def test_poisoned_workspace_gives_the_clean_result(shape, T):
    ex = gpu_experts(shape)
    x = activations(T, shape, seed=34).cuda()
    wr = router_weight(shape).cuda()
    nbytes = moe.forward_workspace_bytes(ex.cfg, T)
    ws0 = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    ws1 = torch.full((nbytes,), 0xFF, dtype=torch.uint8, device="cuda")
    out0, d0 = moe.forward(ex, x, wr, ws=ws0, debug=True)
    assert moe.status_read(ws0) == moe.OK
    out1, d1 = moe.forward(ex, x, wr, ws=ws1, debug=True)
    assert moe.status_read(ws1) == moe.OK
    for key in ("idx", "w", "g_x", "xq_codes", "xq_scales", "counts", "offsets", "perm", "hq_codes", "hq_scales"):
        assert torch.equal(d0[key], d1[key]), key
    assert bool(torch.isfinite(out1.float()).all())
    assert _within_one_bf16_unit(out1, out0)


def test_failed_allocation_leaves_no_error_for_the_next_call():
    """A runtime call that fails inside the library (here the expert weights' allocation for a
    shape far beyond the device's memory: 256 experts of H = I = 32768, 275 GB of codes) returns
    NVFP4MOE_ERR_CUDA and leaves the thread's last CUDA error clear, so neither the library's
    next call nor torch's next launch reports it as its own."""
    ex = gpu_experts(TINY)
    x = activations(16, TINY, seed=35).cuda()
    wr = router_weight(TINY).cuda()
    ws = torch.zeros(moe.forward_workspace_bytes(ex.cfg, 16), dtype=torch.uint8, device="cuda")
    ref = moe.forward(ex, x, wr, ws=ws)
    torch.cuda.synchronize()
    with pytest.raises(moe.NvFp4MoeError) as err:
        moe.Experts(moe.Cfg(256, 8, 4, 8, 32768, 32768, 2.5))
    assert err.value.status == moe.ERR_CUDA
    y = x.clone()                                  # a torch launch right after the failure
    got = moe.forward(ex, y, wr, ws=ws)
    torch.cuda.synchronize()
    assert moe.status_read(ws) == moe.OK
    assert _within_one_bf16_unit(got, ref)
