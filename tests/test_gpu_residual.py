"""The layer fused with its residual-stream neighbours (nvfp4moe_forward_residual) against the
oracle ("Reflection releases Beam ...", section "Residual stream and numerical decisions"):
the normalised layer input bit-exact, the layer on that input under the same protocol as
nvfp4moe_forward (routing near-ties, quantised input bit-exact, grouping), and the updated
residual stream h' = a h + b moe(x) within the output tolerance scaled by b plus its BF16
rounding."""
import numpy as np
import pytest
import torch

import oracle
import nvfp4_quantized_moe_group_b200 as moe
from workloads import TINY, BEAM, activations, router_weight
from tests.helpers import check_routing, intermediate_scales, oracle_layer, bf16_half_ulp
from tests.test_gpu_forward import gpu_experts, check_grouping

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    moe.lib()


def _stream_and_gamma(shape, T, seed):
    """A residual stream of RMS about 3 and a BF16-valued norm weight near 1 (seeded)."""
    h = (activations(T, shape, seed=seed).float() * 3.0).to(torch.bfloat16)
    gen = torch.Generator().manual_seed(1000 + seed)
    gamma = (1.0 + 0.1 * torch.randn(shape.H, generator=gen)).to(torch.bfloat16).float()
    return h, gamma


def run_residual(shape, T, k, tokens=None, in_place=False, eps=1e-6, seed=21):
    ex = gpu_experts(shape)
    h, gamma = _stream_and_gamma(shape, T, seed)
    wr = router_weight(shape)
    ws = torch.empty(moe.forward_workspace_bytes(ex.cfg, T), dtype=torch.uint8, device="cuda")
    h_dev = h.cuda()
    out = h_dev if in_place else None
    h_new, dbg = moe.forward_residual(ex, h_dev, gamma.cuda(), eps, k, wr.cuda(), out=out, ws=ws, debug=True)
    assert moe.status_read(ws) == moe.OK
    if in_place:
        assert h_new.data_ptr() == h_dev.data_ptr()
    hn = h.float().numpy()
    # the normalised layer input: bit-exact
    x_ref = oracle.rmsnorm(hn, gamma.numpy(), eps)
    x_gpu = dbg["x_norm"].float().cpu().numpy()
    np.testing.assert_array_equal(x_gpu, x_ref)
    # the layer on that input
    g_h = intermediate_scales(shape)
    ref = oracle_layer(shape, x_ref, wr.numpy(), None, g_h, tokens=tokens)
    r = ref["route"]
    idx = dbg["idx"].cpu().numpy()
    check_routing(idx, dbg["w"].cpu().numpy(), r, x_ref.astype(np.float64), wr.numpy().astype(np.float64),
                  None, shape)
    assert np.float32(dbg["g_x"].item()) == ref["g_x"]
    np.testing.assert_array_equal(dbg["xq_codes"].cpu().numpy(), ref["xq_codes"])
    check_grouping(dbg, idx, shape.E)
    # the residual update, on tokens routed as the oracle routes them
    toks = ref["tokens"]
    same = np.array([(idx[t] == r.idx[t]).all() for t in toks])
    assert same.sum() >= 1
    a, b = oracle.residual_weights(k)
    want = oracle.residual_add(hn[toks[same]], ref["out"][same], k)
    got = h_new.float().cpu().numpy()[toks[same]]
    err = np.abs(got - want)
    lim = float(b) * 2e-2 + bf16_half_ulp(want) + 1e-6 * np.abs(want)
    assert not (err > lim).any(), f"worst {err.max():.4g}"
    return float(err.max())


def test_tiny_fused_front_end():
    run_residual(TINY, 64, k=5)


def test_tiny_large_batch_in_place():
    run_residual(TINY, 130, k=2, in_place=True)


def test_beam_decode():
    run_residual(BEAM, 16, k=30, tokens=[0, 7, 15])


def test_step_one_is_the_layer_output():
    """k = 1: the stream weight is 0, so h' equals the plain forward on the same input."""
    ex = gpu_experts(TINY)
    T = 24
    h, gamma = _stream_and_gamma(TINY, T, 5)
    wr = router_weight(TINY).cuda()
    h_new, dbg = moe.forward_residual(ex, h.cuda(), gamma.cuda(), 1e-6, 1, wr, debug=True)
    plain = moe.forward(ex, dbg["x_norm"], wr)
    torch.cuda.synchronize()
    diff = (h_new.float() - plain.float()).abs()
    assert bool((diff <= 2.0 ** -7 * plain.float().abs() + 1e-30).all())   # FP32 atomic order


def test_bad_arguments_are_rejected():
    ex = gpu_experts(TINY)
    h, gamma = _stream_and_gamma(TINY, 8, 3)
    wr = router_weight(TINY).cuda()
    for k, eps in ((0, 1e-6), (3, -1.0), (3, float("nan"))):
        with pytest.raises(moe.NvFp4MoeError):
            moe.forward_residual(ex, h.cuda(), gamma.cuda(), eps, k, wr)
