"""Expert parallelism on the CPU: gloo ranks (world size 2 and 4) run ExpertParallelLayer with
the oracle standing in for each rank's partial layer (its share of the tiny layer's 32 experts).
The exchange (all-gather of the tokens, reduce-scatter of the FP32 sums) must give every rank
the oracle's whole-layer output for its own tokens ("Reflection releases Beam ...", section
"Tool calling and multi-node setups": experts placed on the devices, the rest replicated)."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
T_RANK = 8


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import nvfp4_quantized_moe_group_b200 as moe
    from nvfp4_quantized_moe_group_b200.ep import ExpertParallelLayer
    from workloads import TINY, activations, router_weight
    from tests.helpers import oracle_layer, intermediate_scales

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        s = TINY
        cfg = moe.Cfg(s.E, s.n_groups, s.topk_groups, s.topk, s.H, s.I, s.routed_scale)
        wr = router_weight(s)
        g_h = intermediate_scales(s)
        calls = []

        def partial(x_all, w_router, bias):
            calls.append((x_all.shape[0], layer.e_begin, layer.e_count))
            ref = oracle_layer(s, x_all.float().numpy(), w_router.numpy(), None, g_h, workers=1,
                               expert_range=(layer.e_begin, layer.e_count))
            return torch.from_numpy(ref["out"].astype(np.float32))

        layer = ExpertParallelLayer(cfg, partial=partial, finalize=lambda acc: acc.to(torch.bfloat16))
        x = activations(T_RANK, s, seed=40 + rank)
        y = layer.forward(x, wr)
        out[rank] = (layer.e_begin, layer.e_count, calls, y.float().numpy(), x.float().numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_gloo_ranks_expert_parallel_layer(world):
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    sys.path.insert(0, ROOT)
    from workloads import TINY, router_weight
    from tests.helpers import oracle_layer, intermediate_scales, bf16_half_ulp
    # disjoint expert shares covering all experts, each rank called once on all tokens
    n = TINY.E // world
    assert [(res[r][0], res[r][1]) for r in range(world)] == [(r * n, n) for r in range(world)]
    assert all(res[r][2] == [(world * T_RANK, res[r][0], res[r][1])] for r in range(world))
    # every rank's output is the whole layer on its own tokens
    x_all = np.concatenate([res[r][4] for r in range(world)])
    ref = oracle_layer(TINY, x_all, router_weight(TINY).numpy(), None, intermediate_scales(TINY), workers=1)
    for r in range(world):
        want = ref["out"][r * T_RANK:(r + 1) * T_RANK]
        got = res[r][3]
        # FP32 partial sums added across ranks, then BF16: within one BF16 unit of the oracle
        assert np.all(np.abs(got - want) <= 2 * bf16_half_ulp(want) + 1e-30)


def test_expert_range_split():
    sys.path.insert(0, ROOT)
    from nvfp4_quantized_moe_group_b200.ep import expert_range
    assert [expert_range(256, r, 8) for r in range(8)] == [(32 * r, 32) for r in range(8)]
    assert expert_range(256, 0, 1) == (0, 256)
    with pytest.raises(ValueError):
        expert_range(256, 0, 3)
