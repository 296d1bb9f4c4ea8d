"""The FP8 W8A8 variant ("FP8 quantization", section "Quantization scheme") against the oracle:
per-row quantisation bit-exact (codes and scales), the layer's routing under the near-tie
protocol, its per-token quantised input bit-exact, the grouping valid, and the outputs within
max-abs 2e-2 (plus the BF16 output rounding) and relative Frobenius 5e-3 of the oracle's FP64
layer on the same FP8 operands."""
import numpy as np
import pytest
import torch

import oracle
import nvfp4_quantized_moe_group_b200 as moe
from workloads import TINY, BEAM, activations, router_weight, expert_weight
from tests.helpers import check_routing, check_output, oracle_layer_fp8
from tests.test_gpu_forward import check_grouping

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    moe.lib()


_EXPERTS = {}


def gpu_fp8_experts(shape):
    """The layer's experts quantised per output channel on the GPU from the seeded BF16 weights."""
    if shape not in _EXPERTS:
        cfg = moe.make_cfg(shape.E, shape.n_groups, shape.topk_groups, shape.topk, shape.H, shape.I,
                           shape.routed_scale)
        ex = moe.Fp8Experts(cfg)
        for e in range(shape.E):
            ex.set_from_bf16(e, *(expert_weight(shape, e, w, device="cuda") for w in ("gate", "up", "down")))
        torch.cuda.synchronize()
        _EXPERTS[shape] = ex
    return _EXPERTS[shape]


def _rows(rows, cols, seed):
    """Seeded BF16 rows over many magnitudes, with an all-zero row and a row of one value."""
    gen = torch.Generator().manual_seed(seed)
    x = torch.randn(rows, cols, generator=gen) * torch.exp2(torch.randint(-20, 20, (rows, 1), generator=gen).float())
    x[1] = 0.0
    x[2] = -3.0
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("rows,cols", [(1, 16), (37, 80), (300, 5120), (5, 2560)])
def test_quantize_fp8_bit_exact(rows, cols):
    x = _rows(max(rows, 3), cols, seed=rows + cols)
    codes, scales = moe.quantize_fp8(x.cuda())
    ref_c, ref_s = oracle.fp8.quantize_rows(x.float().numpy())
    np.testing.assert_array_equal(scales.cpu().numpy(), ref_s)
    np.testing.assert_array_equal(codes.cpu().numpy(), ref_c)


def test_quantize_fp8_division_tie_and_negative_zero():
    """A value whose FP32 quotient v / s is exactly the E4M3 midpoint 5.25 (the tie goes to the
    even code 0x4A; a multiply by fp32(1 / s) would land above it and give 0x4B), and signed
    zeros (-0 keeps its sign bit, 0x80), bit-exact against the oracle."""
    x = torch.zeros(2, 16)
    x[0, :4] = torch.tensor([1.078125, 0.01263427734375, -0.0, 0.0])
    x[1, :4] = torch.tensor([-1.078125, -0.01263427734375, 0.0, -0.0])
    x = x.to(torch.bfloat16)
    codes, scales = moe.quantize_fp8(x.cuda())
    ref_c, ref_s = oracle.fp8.quantize_rows(x.float().numpy())
    assert list(ref_c[0, :4]) == [0x7E, 0x4A, 0x80, 0x00]
    np.testing.assert_array_equal(scales.cpu().numpy(), ref_s)
    np.testing.assert_array_equal(codes.cpu().numpy(), ref_c)


def test_quantize_fp8_expert_weights_bit_exact():
    """The weights the layer uses: the GPU's per-channel codes and scales equal the oracle's."""
    for w in ("gate", "down"):
        wt = expert_weight(BEAM, 3, w)
        codes, scales = moe.quantize_fp8(wt.cuda())
        t = oracle.fp8.Fp8Tensor(wt.float().numpy())
        np.testing.assert_array_equal(scales.cpu().numpy(), t.scales)
        np.testing.assert_array_equal(codes.cpu().numpy(), t.codes)


def test_quantize_fp8_nonfinite_row_raises_status():
    x = _rows(8, 64, seed=3)
    x[5, 7] = float("inf")
    ws = torch.empty(moe.quantize_workspace_bytes(8, 64), dtype=torch.uint8, device="cuda")
    codes, scales = moe.quantize_fp8(x.cuda(), ws=ws)
    assert moe.status_read(ws) == moe.ERR_NONFINITE
    ref_c, ref_s = oracle.fp8.quantize_rows(np.delete(x.float().numpy(), 5, axis=0))
    keep = [r for r in range(8) if r != 5]
    np.testing.assert_array_equal(codes.cpu().numpy()[keep], ref_c)
    np.testing.assert_array_equal(scales.cpu().numpy()[keep], ref_s)


def run_layer_fp8(shape, T, tokens=None, rms_rows=False):
    ex = gpu_fp8_experts(shape)
    x = activations(T, shape, rms_rows=rms_rows)
    wr = router_weight(shape)
    ws = torch.empty(moe.forward_fp8_workspace_bytes(ex.cfg, T), dtype=torch.uint8, device="cuda")
    out, dbg = moe.forward_fp8(ex, x.cuda(), wr.cuda(), ws=ws, debug=True)
    assert moe.status_read(ws) == moe.OK
    xn = x.float().numpy()
    ref = oracle_layer_fp8(shape, xn, wr.numpy(), None, tokens=tokens)
    r = ref["route"]
    idx = dbg["idx"].cpu().numpy()
    check_routing(idx, dbg["w"].cpu().numpy(), r, xn.astype(np.float64), wr.numpy().astype(np.float64), None,
                  shape)
    np.testing.assert_array_equal(dbg["xq8_scales"].cpu().numpy(), ref["xq_scales"])
    np.testing.assert_array_equal(dbg["xq8_codes"].cpu().numpy(), ref["xq_codes"])
    check_grouping(dbg, idx, shape.E)
    toks = ref["tokens"]
    same = np.array([(idx[t] == r.idx[t]).all() for t in toks])
    assert same.sum() >= 1
    gpu = out.float().cpu().numpy()[toks[same]]
    return check_output(gpu, ref["out"][same], bf16=True)


def test_tiny_layer_all_tokens():
    run_layer_fp8(TINY, 64)


def test_tiny_layer_ragged_and_single():
    for T in (1, 5, 130):
        run_layer_fp8(TINY, T)


def test_beam_decode_layer():
    run_layer_fp8(BEAM, 16, tokens=[0, 11], rms_rows=True)


def test_beam_prefill_layer_sampled():
    """Full expert segments (the staged down-projection epilogue)."""
    run_layer_fp8(BEAM, 4096, tokens=[0, 4095])


def test_forward_fp8_launch_count_and_bad_arguments():
    ex = gpu_fp8_experts(TINY)
    x = activations(8, TINY).cuda()
    wr = router_weight(TINY).cuda()
    moe.forward_fp8(ex, x, wr)
    assert moe.last_launch_count() == 1 + 5          # fused front end, then the FP8 stages
    moe.forward_fp8(ex, activations(600, TINY).cuda(), wr)
    assert moe.last_launch_count() == 4 + 4 + 5      # integer router, 4-kernel grouping, FP8 stages
    ws = torch.empty(64, dtype=torch.uint8, device="cuda")
    with pytest.raises(moe.NvFp4MoeError):
        moe.forward_fp8(ex, x, wr, ws=ws)
