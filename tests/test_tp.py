"""Tensor parallelism on the CPU (the checkpoint is validated with four-way tensor parallelism:
"NVFP4 quantization", section "Hardware compatibility and serving").

Rank r of G holds features [r I/G, (r+1) I/G) of every expert, cut from the whole tensors'
quantisation.  Checked here without a GPU: the split of I, that the cut codes and scales
dequantise to the matching slice of the whole tensor, that the oracle's layer summed over the
slices equals its whole layer (the reading that the slices are the single-GPU operands of
their features), and gloo ranks (world 2 and 4) running TensorParallelLayer with the oracle
standing in for the library's partial call."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from nvfp4_quantized_moe_group_b200.tp import intermediate_range, slice_expert
from workloads import LayerShape, activations, expert_weight, router_weight
from tests.helpers import cfg_ns

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# the tiny layer with an intermediate size that splits into 4 slices of 128 features
TP_SHAPE = LayerShape(H=256, I=512, E=32, n_groups=8, topk_groups=4, topk=8, routed_scale=2.5,
                      wr_std=1.0 / 16.0, w_std=0.02)
T = 12


def _g_h(shape):
    return (np.float32(0.004) * (1 + np.arange(shape.E, dtype=np.float32) / shape.E)).astype(np.float32)


def _whole_expert(shape, e):
    return tuple(oracle.quantize(expert_weight(shape, e, w).float().numpy()) for w in ("gate", "up", "down"))


def _sliced_expert(whole, i0, n):
    """The rank's slice through the package's slicing, as oracle tensors."""
    t = [(torch.from_numpy(c), torch.from_numpy(s), float(g)) for c, s, g in whole]
    return tuple(oracle.QuantTensor(c.numpy(), s.numpy(), np.float32(g)) for c, s, g in slice_expert(*t, i0, n))


def test_intermediate_range():
    assert [intermediate_range(2560, r, 4) for r in range(4)] == [(0, 640), (640, 640), (1280, 640), (1920, 640)]
    assert intermediate_range(2560, 1, 2) == (1280, 1280)
    assert intermediate_range(2560, 0, 1) == (0, 2560)
    for I, world in ((2560, 8), (2560, 3), (128, 2), (512, 0)):
        with pytest.raises(ValueError):
            intermediate_range(I, 0, world)


@pytest.mark.parametrize("world", [2, 4])
def test_slices_dequantise_to_the_whole_tensors_slices(world):
    whole = _whole_expert(TP_SHAPE, 5)
    full = [oracle.dequantize(*w) for w in whole]
    for r in range(world):
        i0, n = intermediate_range(TP_SHAPE.I, r, world)
        g, u, d = _sliced_expert(whole, i0, n)
        assert g.g == whole[0][2] and u.g == whole[1][2] and d.g == whole[2][2]
        np.testing.assert_array_equal(g.dequant(), full[0][i0:i0 + n])
        np.testing.assert_array_equal(u.dequant(), full[1][i0:i0 + n])
        np.testing.assert_array_equal(d.dequant(), full[2][:, i0:i0 + n])


def test_slice_must_keep_blocks_whole():
    whole = [(torch.zeros(64, 8, dtype=torch.uint8), torch.zeros(64, 1, dtype=torch.uint8), 1.0)] * 2
    down = (torch.zeros(16, 32, dtype=torch.uint8), torch.zeros(16, 4, dtype=torch.uint8), 1.0)
    with pytest.raises(ValueError):
        slice_expert(whole[0], whole[1], down, 8, 32)


def _oracle_out(x, wr, experts, g_h):
    return oracle.moe_forward(x, wr, cfg_ns(TP_SHAPE), experts, g_h)["out"]


@pytest.mark.parametrize("world", [2, 4])
def test_layer_is_the_sum_over_the_slices(world):
    """Routing and the input quantisation do not depend on I; each feature's SwiGLU product and
    its requantisation (blocks of 16 features) depend on that feature alone; the down
    projection is a sum over features.  So the layer is the sum of the slices' layers, up to
    the order of the FP64 additions."""
    x = activations(T, TP_SHAPE, seed=3).float().numpy()
    wr = router_weight(TP_SHAPE).numpy()
    g_h = _g_h(TP_SHAPE)
    whole = {e: _whole_expert(TP_SHAPE, e) for e in range(TP_SHAPE.E)}
    want = _oracle_out(x, wr, lambda e: tuple(oracle.QuantTensor(*w) for w in whole[e]), g_h)
    got = np.zeros_like(want)
    for r in range(world):
        i0, n = intermediate_range(TP_SHAPE.I, r, world)
        got += _oracle_out(x, wr, lambda e: _sliced_expert(whole[e], i0, n), g_h)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-15 * np.abs(want).max())


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import nvfp4_quantized_moe_group_b200 as moe
    from nvfp4_quantized_moe_group_b200.tp import TensorParallelLayer

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        s = TP_SHAPE
        cfg = moe.Cfg(s.E, s.n_groups, s.topk_groups, s.topk, s.H, s.I, s.routed_scale)
        g_h = _g_h(s)
        whole = {e: _whole_expert(s, e) for e in range(s.E)}
        calls = []

        def partial(x, w_router, bias):
            calls.append((x.shape[0], layer.i0, layer.n, layer.cfg_local.I))
            res = _oracle_out(x.float().numpy(), w_router.numpy(),
                              lambda e: _sliced_expert(whole[e], layer.i0, layer.n), g_h)
            return torch.from_numpy(res)              # FP64: the exchange is what is checked

        layer = TensorParallelLayer(cfg, partial=partial, finalize=lambda acc: acc)
        x = activations(T, s, seed=3)                 # the same tokens on every rank
        y = layer.forward(x, router_weight(s))
        out[rank] = (calls, y.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_gloo_ranks_tensor_parallel_layer(world):
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    n = TP_SHAPE.I // world
    # each rank called once on all tokens with its own slice of every expert
    assert [res[r][0] for r in range(world)] == [[(T, r * n, n, n)] for r in range(world)]
    x = activations(T, TP_SHAPE, seed=3).float().numpy()
    whole = {e: _whole_expert(TP_SHAPE, e) for e in range(TP_SHAPE.E)}
    want = _oracle_out(x, router_weight(TP_SHAPE).numpy(),
                       lambda e: tuple(oracle.QuantTensor(*w) for w in whole[e]), _g_h(TP_SHAPE))
    for r in range(world):
        # the all-reduced sums: the whole layer on every rank
        np.testing.assert_allclose(res[r][1], want, rtol=1e-12, atol=1e-15 * np.abs(want).max())
        np.testing.assert_array_equal(res[r][1], res[0][1])
