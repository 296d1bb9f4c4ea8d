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


def _run(shape, T, rms_rows=False, bias=None, max_flag_frac=0.1, bf16_router=False):
    x = activations(T, shape, rms_rows=rms_rows)
    wr = router_weight(shape)
    if bf16_router:
        wr = wr.bfloat16().float()
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


@pytest.mark.parametrize("T", [16, 4096])
def test_bf16_valued_router_weights(T):
    """A router kept in BF16 (the quantisation page leaves routers in BF16) is the special case
    of FP32 router rows whose values are BF16: both logit paths (T <= 64 and the integer one)
    route it under the same protocol."""
    _run(BEAM, T, rms_rows=T == 16, bf16_router=True)


def test_ragged_token_counts():
    for T in (3, 65, 130):
        _run(BEAM, T)


# Group layouts beyond Beam's: group sizes that are not a power of two (the in-group ranks
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
    # groups of one and two lanes of the warp-per-token top-k, and a group of 24 experts
    # (three lanes: not a butterfly, so the block top-k takes it)
    "gs8": LayerShape(H=256, I=128, E=64, n_groups=8, topk_groups=3, topk=8, routed_scale=2.5,
                      wr_std=1.0 / 16.0, w_std=0.02),
    "gs16": LayerShape(H=256, I=128, E=128, n_groups=8, topk_groups=2, topk=6, routed_scale=2.5,
                       wr_std=1.0 / 16.0, w_std=0.02),
    "gs24": LayerShape(H=256, I=128, E=96, n_groups=4, topk_groups=2, topk=8, routed_scale=2.5,
                       wr_std=1.0 / 16.0, w_std=0.02),
}


@pytest.mark.parametrize("name", sorted(ODD_SHAPES))
@pytest.mark.parametrize("T", [16, 100])
def test_group_layouts(name, T):
    _run(ODD_SHAPES[name], T)


@pytest.mark.parametrize("T", [16, 512])
def test_exact_ties_go_to_the_lower_index(T):
    """Router rows duplicated on purpose (expert 5 = expert 4, scaled up so that the pair is
    often selected; every expert of group 3 = its counterpart in group 2) give bit-identical
    logits on every path, so the tie rules decide:
    a token never takes expert 5 without expert 4, nor group 3 without group 2, equal experts
    are listed lower index first, and their weights are equal.  nvfp4moe_route (FP32 logits at
    T = 16, tensor-core logits at T = 512, both with the warp-per-token top-k), the
    allocation-free router (FP32 logits) and, at T = 16, the forward's fused front end (its
    block top-k) are checked on the same rows."""
    shape = BEAM
    cfg = moe.make_cfg(shape.E, shape.n_groups, shape.topk_groups, shape.topk, shape.H, shape.I,
                       shape.routed_scale)
    wr = router_weight(shape).clone()
    wr[4] = 3.0 * wr[4]                     # a larger logit spread: expert 4 is picked often
    wr[5] = wr[4]
    wr[96:128] = wr[64:96]
    x = activations(T, shape, seed=17).cuda()
    runs = {"route": moe.route(cfg, x, wr.cuda()), "route_noalloc": moe.route_noalloc(cfg, x, wr.cuda())}
    if T <= 64:
        from tests.test_gpu_forward import gpu_experts
        _, dbg = moe.forward(gpu_experts(shape), x, wr.cuda(), debug=True)
        runs["forward front end"] = (dbg["idx"], dbg["w"])
    torch.cuda.synchronize()
    n_tie_decided = n_pair = n_group = 0
    for name, (idx, w) in runs.items():
        idx, w = idx.cpu().numpy(), w.cpu().numpy()
        for t in range(T):
            sel = list(idx[t])
            n_pair += 4 in sel
            n_group += any(64 <= e < 128 for e in sel)
            if 5 in sel:
                assert 4 in sel, f"{name} token {t}: expert 5 without expert 4"
                i4, i5 = sel.index(4), sel.index(5)
                assert i5 == i4 + 1, f"{name} token {t}: equal experts 4, 5 not adjacent in index order"
                assert w[t, i4] == w[t, i5]
            elif 4 in sel:
                n_tie_decided += 1
            g3 = [e for e in sel if 96 <= e < 128]
            for e in g3:
                assert e - 32 in sel, f"{name} token {t}: expert {e} of group 3 without its twin {e - 32}"
                assert sel.index(e - 32) < sel.index(e)
    print(f"T={T}: expert 4 selected {n_pair} times ({n_tie_decided} without its twin), groups 2/3 in {n_group}")
    assert n_pair > 0 and n_group > 0
