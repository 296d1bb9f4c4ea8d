"""Router on the GPU against the FP64 oracle under the near-tie protocol: experts and their
order bit-exact wherever the decision margins exceed the documented FP32 error bound,
admissible selections elsewhere, weights to a relative 2e-6."""
import numpy as np
import pytest
import torch

import oracle
import nvfp4_quantized_moe_group_b200 as moe
from workloads import TINY, BEAM, LayerShape, activations, router_weight, zipf_bias
from tests.helpers import cfg_ns, check_routing

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    moe.lib()


def _run(shape, T, rms_rows=False, bias=None, max_flag_frac=0.1):
    x = activations(T, shape, rms_rows=rms_rows)
    wr = router_weight(shape)
    cfg = moe.make_cfg(shape.E, shape.n_groups, shape.topk_groups, shape.topk, shape.H, shape.I,
                       shape.routed_scale)
    idx, w = moe.route(cfg, x.cuda(), wr.cuda(), None if bias is None else bias.cuda())
    torch.cuda.synchronize()
    xn = x.float().numpy().astype(np.float64)
    bn = None if bias is None else bias.numpy()
    r = oracle.route(xn, wr.numpy(), cfg_ns(shape), bn)
    clean, n_flag = check_routing(idx.cpu().numpy(), w.cpu().numpy(), r, xn, wr.numpy().astype(np.float64),
                                  bn, shape)
    assert n_flag <= max_flag_frac * T + 2
    return idx, clean


def test_tiny_layer():
    _, clean = _run(TINY, 64)
    assert clean.all()


def test_beam_decode():
    _run(BEAM, 16, rms_rows=True)


def test_beam_single_token():
    _run(BEAM, 1)


def test_beam_prefill_all_tokens():
    _run(BEAM, 4096)


def test_beam_skewed_zipf_bias():
    idx, _ = _run(BEAM, 16384, bias=zipf_bias(256))
    counts = np.bincount(idx.cpu().numpy().ravel(), minlength=256)
    assert counts.max() > 8 * counts.mean()           # the bias concentrates the load


def test_ragged_token_counts():
    for T in (3, 65, 130):
        _run(BEAM, T)


# Group layouts beyond Beam's: a group size that is not a power of two (the in-group ranks
# go through shared memory instead of shuffles), one expert per group (the group score is
# its single score), every group kept, and more than 32 selection candidates.
ODD_SHAPES = {
    "gs12": LayerShape(H=256, I=128, E=48, n_groups=4, topk_groups=2, topk=6, routed_scale=2.5,
                       wr_std=1.0 / 16.0, w_std=0.02),
    "gs1": LayerShape(H=256, I=128, E=8, n_groups=8, topk_groups=4, topk=3, routed_scale=1.0,
                      wr_std=1.0 / 16.0, w_std=0.02),
    "all_groups": LayerShape(H=256, I=128, E=64, n_groups=2, topk_groups=2, topk=8, routed_scale=2.5,
                             wr_std=1.0 / 16.0, w_std=0.02),
    "64_candidates": LayerShape(H=512, I=128, E=256, n_groups=8, topk_groups=8, topk=8, routed_scale=2.5,
                                wr_std=512 ** -0.5, w_std=0.02),
}


@pytest.mark.parametrize("name", sorted(ODD_SHAPES))
@pytest.mark.parametrize("T", [16, 100])
def test_group_layouts(name, T):
    _run(ODD_SHAPES[name], T)
