"""quantize_nvfp4 on the GPU against the oracle: codes, block scales (both layouts) and the
global scale must be identical bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import nvfp4_quantized_moe_group_b200 as moe
from workloads import BEAM, activations, approx_normal, expert_weight

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    moe.lib()


def _varied(rows, cols, seed):
    """Rows of very different magnitudes, a zero block, a negative-zero block, a tiny block."""
    x = approx_normal((rows, cols), seed, 40, dtype=torch.float32)
    scale = torch.exp(approx_normal((rows, 1), seed, 41, 2.0, dtype=torch.float32))
    x = x * scale
    if rows > 3 and cols >= 64:
        x[1, 16:32] = 0.0
        x[2, 0:16] = -0.0
        x[3, 32:48] *= 1e-6
    return x.to(torch.bfloat16)


def _check(x_bf16, g=None, swizzled=False):
    xc = x_bf16.cuda()
    gt = None if g is None else torch.tensor([g], dtype=torch.float32, device="cuda")
    codes, scales, g_out = moe.quantize(xc, gt, swizzled=swizzled)
    torch.cuda.synchronize()
    oc, os_, og = oracle.quantize(x_bf16.float().numpy(), g=None if g is None else np.float32(g))
    assert np.float32(g_out.item()) == og
    np.testing.assert_array_equal(codes.cpu().numpy(), oc)
    if swizzled:
        np.testing.assert_array_equal(scales.cpu().numpy(), oracle.swizzle_scales(os_))
    else:
        np.testing.assert_array_equal(scales.cpu().numpy(), os_)


@pytest.mark.parametrize("rows,cols", [(1, 64), (7, 256), (129, 5120), (300, 64), (256, 2560), (1000, 320)])
@pytest.mark.parametrize("swizzled", [False, True])
def test_dynamic_scale_bit_exact(rows, cols, swizzled):
    _check(_varied(rows, cols, rows * 7 + cols), swizzled=swizzled)


@pytest.mark.parametrize("g", [0.01, 3.0e-5, 1.0])
def test_static_scale_bit_exact_including_saturation(g):
    _check(_varied(64, 512, 3), g=g)
    _check(_varied(200, 256, 4), g=g, swizzled=True)


def test_expert_weight_tensors_bit_exact():
    for which in ("gate", "down"):
        _check(expert_weight(BEAM, 5, which))


def test_empty_tensor_gives_unit_scale():
    x = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    codes, scales, g = moe.quantize(x, swizzled=True)
    torch.cuda.synchronize()
    assert g.item() == 1.0 and codes.numel() == 0 and scales.numel() == 0


def test_nonfinite_input_sets_status():
    x = _varied(16, 128, 9).cuda()
    x[3, 5] = float("nan")
    ws = torch.empty(moe.quantize_workspace_bytes(16, 128), dtype=torch.uint8, device="cuda")
    moe.quantize(x, ws=ws)
    assert moe.status_read(ws) == moe.ERR_NONFINITE
    moe.quantize(x.nan_to_num(), ws=ws)
    assert moe.status_read(ws) == moe.OK


def test_full_size_activation_sampled_rows():
    """32768 x 5120 BF16 N(0,1) (the standalone quantize workload): the GPU quantises the
    whole tensor; the oracle's global scale comes from its own pass over the CPU copy and
    sampled rows are checked bit for bit (rows are independent once g is fixed)."""
    T = 32768
    x_gpu = activations(T, BEAM, device="cuda")
    codes, scales, g = moe.quantize(x_gpu, swizzled=True)
    torch.cuda.synchronize()
    x_cpu = activations(T, BEAM).float().numpy()
    og = oracle.global_scale(np.abs(x_cpu).max())
    assert np.float32(g.item()) == og
    rows = np.unique(np.concatenate([[0, 1, 127, 128, 4095, 4096, T - 1],
                                     np.random.default_rng(0).integers(0, T, 64)]))
    oc, os_, _ = oracle.quantize(x_cpu[rows], g=og)
    np.testing.assert_array_equal(codes[torch.from_numpy(rows).cuda()].cpu().numpy(), oc)
    sw = scales.cpu().numpy()
    n_ct = 5120 // 64
    for i, r in enumerate(rows):
        c = np.arange(320)
        off = (r // 128) * n_ct * 512 + (c // 4) * 512 + (r % 32) * 16 + (r % 128 // 32) * 4 + c % 4
        np.testing.assert_array_equal(sw[off], os_[i])


def test_generator_same_bits_on_gpu():
    a = approx_normal((1000, 333), 2, 5, 0.7, device="cuda").cpu()
    b = approx_normal((1000, 333), 2, 5, 0.7)
    assert torch.equal(a, b)
