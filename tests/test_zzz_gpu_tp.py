"""Tensor parallelism on one GPU: the ranks' calls run one after another, each with its slice of
every expert's intermediate features (nvfp4_quantized_moe_group_b200.tp), and their FP32 sums
are added on the host as the all-reduce would.  Checked through the C ABI against the
single-GPU handle on the same whole-tensor quantisation: every rank routes identically, its
requantised SwiGLU intermediate is bit for bit the matching feature slice of the single-GPU
one, and the ranks' sums add up to the single-GPU sums up to FP32 rounding.  A layer with
Beam's intermediate size (2560: slices of 1280 and 640 features, the latter giving the down
GEMM a last K block of 128 values) and a smaller hidden size, at a decode-regime and a
full-segment token count ("NVFP4 quantization", section "Hardware compatibility and serving":
four-way tensor parallelism)."""
import numpy as np
import pytest
import torch

import nvfp4_quantized_moe_group_b200 as moe
from nvfp4_quantized_moe_group_b200.tp import intermediate_range, slice_expert
from workloads import LayerShape, activations, expert_weight, router_weight
from tests.helpers import bf16_half_ulp

pytestmark = pytest.mark.gpu

SHAPE = LayerShape(H=512, I=2560, E=16, n_groups=4, topk_groups=2, topk=4, routed_scale=2.5,
                   wr_std=512 ** -0.5, w_std=0.02)
_WHOLE = {}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    moe.lib()


def _cfg(I):
    s = SHAPE
    return moe.make_cfg(s.E, s.n_groups, s.topk_groups, s.topk, s.H, I, s.routed_scale)


def _whole_experts():
    """Every expert's whole-tensor quantisation on the GPU (codes, linear scales, global
    scale) and a static intermediate scale per expert."""
    if not _WHOLE:
        for e in range(SHAPE.E):
            q = []
            for w in ("gate", "up", "down"):
                c, s, g = moe.quantize(expert_weight(SHAPE, e, w, device="cuda"))
                q.append((c, s, float(g.item())))
            _WHOLE[e] = tuple(q)
        _WHOLE["g_h"] = [0.001 * (1 + e / SHAPE.E) for e in range(SHAPE.E)]
    return _WHOLE


def _handle(I, i0=0):
    whole = _whole_experts()
    ex = moe.Experts(_cfg(I))
    for e in range(SHAPE.E):
        parts = whole[e] if I == SHAPE.I else slice_expert(*whole[e], i0, I)
        ex.set(e, *parts, whole["g_h"][e])
    torch.cuda.synchronize()
    return ex


@pytest.mark.parametrize("world,T", [(2, 64), (4, 64), (2, 600), (4, 600)])
def test_ranks_add_up_to_the_single_gpu_layer(world, T):
    single = _handle(SHAPE.I)
    x = activations(T, SHAPE, seed=60).cuda()
    wr = router_weight(SHAPE).cuda()
    acc_full, dbg = moe.forward_partial(single, x, wr, debug=True)
    out_full = moe.forward(single, x, wr)
    torch.cuda.synchronize()
    total = torch.zeros_like(acc_full)
    for r in range(world):
        i0, n = intermediate_range(SHAPE.I, r, world)
        ex = _handle(n, i0)
        acc_r, dbg_r = moe.forward_partial(ex, x, wr, debug=True)
        torch.cuda.synchronize()
        assert torch.equal(dbg_r["idx"], dbg["idx"]), f"rank {r} routes differently"
        assert torch.equal(dbg_r["xq_codes"], dbg["xq_codes"]) and torch.equal(dbg_r["g_x"], dbg["g_x"])
        # a feature's SwiGLU product and its requantisation depend on that feature alone
        assert torch.equal(dbg_r["hq_codes"], dbg["hq_codes"][:, i0 // 2:(i0 + n) // 2]), f"rank {r}: h codes"
        assert torch.equal(dbg_r["hq_scales"], dbg["hq_scales"][:, i0 // 16:(i0 + n) // 16]), f"rank {r}: h scales"
        total += acc_r
        ex.close()
    af = acc_full.cpu().numpy()
    diff = np.abs(total.cpu().numpy() - af)
    # the same products summed over K in slices: FP32 roundings of the partial sums, far below
    # one slice's whole contribution
    row_scale = np.abs(af).max(axis=1, keepdims=True)
    assert np.all(diff <= 2.0 ** -12 * row_scale + 1e-30), f"max diff/row scale {np.max(diff / (row_scale + 1e-30)):.3g}"
    out_tp = moe.finalize(total).float().cpu().numpy()
    of = out_full.float().cpu().numpy()
    bad = np.abs(out_tp - of) > 2 * bf16_half_ulp(of) + 2.0 ** -12 * np.abs(of).max(axis=1, keepdims=True) + 1e-30
    assert not bad.any(), f"{int(bad.sum())} outputs beyond one BF16 unit"
    single.close()
