"""The local-Hessian block-scale search on the GPU (nvfp4moe_quantize_weights_lh) against the
oracle ("NVFP4 quantization", section "Quantization method").  The oracle evaluates every
candidate's error in FP64, the kernel in FP32: where the best candidate wins by more than a
relative 1e-4 the GPU must pick it; elsewhere it must pick a candidate within that margin of
the best.  For the scale it picked, its codes must equal the quantisation rule's bit for bit.
With no extra candidates (m = 0) it must reproduce nvfp4moe_quantize exactly."""
import numpy as np
import pytest
import torch

import oracle
import nvfp4_quantized_moe_group_b200 as moe
from oracle.local_hessian import codes_for_scale
from workloads.synthetic import approx_normal

pytestmark = pytest.mark.gpu

MARGIN = 1e-4


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    moe.lib()


def _case(rows, cols, n_cal, seed):
    """BF16 weights (std 0.02) and the local Hessian blocks of correlated calibration inputs."""
    w = (approx_normal((rows, cols), seed, 41, 0.02)).to(torch.bfloat16)
    z = approx_normal((n_cal, cols), seed, 42, 1.0).double().numpy()
    mix = approx_normal((cols,), seed, 43, 1.0).double().numpy()
    x = z + 0.5 * np.roll(z, 1, axis=1) * mix[None, :]      # neighbouring inputs correlate
    return w, oracle.hessian_blocks(x)


def _gpu(w, H, m):
    codes, scales, g = moe.quantize_weights_lh(w.cuda(), torch.from_numpy(H.astype(np.float32)).cuda(), m)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy(), np.float32(g.item())


@pytest.mark.parametrize("rows,cols,m", [(256, 512, 4), (300, 256, 2), (64, 5120, 4)])
def test_search_matches_oracle(rows, cols, m):
    w, H = _case(rows, cols, 128, seed=rows + cols)
    wf = w.float().numpy()
    codes, S, g = _gpu(w, H, m)
    c_ref, S_ref, g_ref, errs, cands = oracle.quantize_local_hessian(wf, H.astype(np.float32).astype(np.float64), m)
    assert g == g_ref
    best = errs.min(axis=2)
    # index of the GPU's scale among the candidates
    hit = cands == S[..., None].astype(np.int64)
    assert hit.any(axis=2).all()
    k_gpu = np.argmax(hit, axis=2)
    e_gpu = np.take_along_axis(errs, k_gpu[..., None], axis=2)[..., 0]
    assert np.all(e_gpu <= best * (1 + MARGIN) + 1e-30)
    # where the oracle's choice wins clearly, the same scale
    second = np.sort(errs, axis=2)[..., 1] if errs.shape[2] > 1 else np.full_like(best, np.inf)
    distinct = np.array([[len(set(c)) for c in row] for row in cands])
    clear = (second > best * (1 + MARGIN)) | (distinct == 1)
    np.testing.assert_array_equal(S[clear], S_ref[clear])
    assert clear.mean() > 0.95
    # codes of the scale the GPU picked: the quantisation rule exactly
    c_gpu = codes_for_scale(wf.reshape(rows, cols // 16, 16), S, g).reshape(rows, cols)
    np.testing.assert_array_equal(codes, (c_gpu[:, 0::2] | (c_gpu[:, 1::2] << 4)).astype(np.uint8))


def test_no_candidates_is_plain_quantisation():
    w, H = _case(128, 1024, 64, seed=5)
    codes, S, g = _gpu(w, H, 0)
    c_ref, s_ref, g_ref = moe.quantize(w.cuda())
    torch.cuda.synchronize()
    np.testing.assert_array_equal(codes, c_ref.cpu().numpy())
    np.testing.assert_array_equal(S, s_ref.cpu().numpy())
    assert g == np.float32(g_ref.item())


def test_worked_block_on_gpu():
    """The hand-built block of the oracle pins: scale 11 (code 83) represents 2.75 exactly."""
    w = torch.zeros((2, 16), dtype=torch.bfloat16)
    w[0, 0] = 168.0
    w[1, 0] = 2.75
    H = np.zeros((1, 16, 16))
    H[0, 0, 0] = 1.0
    codes, S, g = _gpu(w, H, 4)
    assert g == np.float32(1 / 16)
    assert S[1, 0] == 83


def test_bad_arguments_are_rejected():
    w = torch.zeros((4, 24), dtype=torch.bfloat16).cuda()          # cols not a multiple of 16
    with pytest.raises(moe.NvFp4MoeError):
        moe.quantize_weights_lh(w, torch.zeros((1, 16, 16)).cuda(), 4)
    w = torch.zeros((4, 32), dtype=torch.bfloat16).cuda()
    with pytest.raises(moe.NvFp4MoeError):
        moe.quantize_weights_lh(w, torch.zeros((2, 16, 16)).cuda(), 17)
