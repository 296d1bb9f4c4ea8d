"""Expert parallelism on the CPU: gloo ranks (world size 2 and 4) run ExpertParallelLayer with
the oracle standing in for the library's calls (each rank's share of the tiny layer's 32
experts).  Both exchanges (all-gather of the tokens with a reduce-scatter of the FP32 sums;
all-to-all of the pairs' quantised rows and of their weighted output rows) must give every
rank the oracle's whole-layer output for its own tokens ("Reflection releases Beam ...", section
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


def _rank_main_a2a(rank, world, port, out):
    """One gloo rank of the all-to-all exchange, the library's four calls replaced by oracle
    stand-ins (routing, quantisation with the global scale, grouping, expert MLPs, slot-order
    combine), kept in FP64 so the exchange itself is what the comparison checks."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import oracle
    import nvfp4_quantized_moe_group_b200 as moe
    from nvfp4_quantized_moe_group_b200.ep import ExpertParallelLayer
    from workloads import TINY, activations, router_weight
    from tests.helpers import cfg_ns, intermediate_scales, oracle_expert

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        s = TINY
        cfg = moe.Cfg(s.E, s.n_groups, s.topk_groups, s.topk, s.H, s.I, s.routed_scale)
        g_h = intermediate_scales(s)
        k = s.topk
        seen = {}

        def g_of(amax_bits):
            a = np.array([int(amax_bits.item()) << 16], dtype=np.uint32).view(np.float32)[0]
            return oracle.global_scale(a)

        def amax(x):
            return (x.view(torch.int16).to(torch.int32) & 0x7FFF).max().reshape(1)

        def dispatch(x, wr, bias, amax_bits):
            xn = x.float().numpy()
            r = oracle.route(xn.astype(np.float64), wr.numpy().astype(np.float64), cfg_ns(s), None)
            codes, scales, _ = oracle.quantize(xn, g=g_of(amax_bits))
            counts, _, perm, inv = oracle.permutation(r.idx, s.E)
            epr = s.E // world
            seen["send_counts"] = counts.reshape(world, epr).sum(axis=1).tolist()
            return {"codes": torch.from_numpy(codes[perm // k]), "scales": torch.from_numpy(scales[perm // k]),
                    "expert": torch.from_numpy((r.idx.reshape(-1)[perm] % epr).astype(np.int32)),
                    "w": torch.from_numpy(r.w.reshape(-1)[perm].astype(np.float64)),
                    "pos": torch.from_numpy(inv.reshape(-1).astype(np.int32)),
                    "rank_counts": torch.from_numpy(counts.reshape(world, epr).sum(axis=1).astype(np.int32))}

        def experts(codes, scales, expert, w, amax_bits):
            seen["recv_rows"] = int(codes.shape[0])
            xhat = oracle.dequantize(codes.numpy(), scales.numpy(), g_of(amax_bits))
            rows = np.zeros((codes.shape[0], s.H))
            e_loc = expert.numpy()
            for e in np.unique(e_loc):
                sel = np.flatnonzero(e_loc == e)
                eg = int(e) + layer.e_begin
                y = oracle.expert_mlp(xhat[sel], *oracle_expert(s, eg), np.float32(g_h[eg]))["y"]
                rows[sel] = w.numpy()[sel][:, None] * y
            return torch.from_numpy(rows)

        def combine(back, pos, T):
            b = back.numpy()
            p = pos.numpy().reshape(T, k)
            outv = np.zeros((T, s.H))
            for j in range(k):
                outv += b[p[:, j]]
            return torch.from_numpy(outv)

        layer = ExpertParallelLayer(cfg, exchange="all_to_all",
                                    a2a_ops={"amax": amax, "dispatch": dispatch, "experts": experts,
                                             "combine": combine})
        wr = router_weight(s)
        x = activations(T_RANK, s, seed=60 + rank)
        y = layer.forward(x, wr)
        out[rank] = (layer.e_begin, layer.e_count, seen, y.numpy(), x.float().numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_gloo_ranks_all_to_all_exchange(world):
    """The all-to-all exchange on gloo ranks: uneven per-rank counts, rows and their metadata
    out, weighted output rows back, each token's rows added in slot order.  Every rank must get
    the oracle's whole layer on the concatenated batch for its own tokens (the global scale of
    all ranks' tokens included), and the rows each rank receives must be the pairs routed to
    its experts."""
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main_a2a, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    sys.path.insert(0, ROOT)
    from workloads import TINY, router_weight
    from tests.helpers import oracle_layer, intermediate_scales
    x_all = np.concatenate([res[r][4] for r in range(world)])
    ref = oracle_layer(TINY, x_all, router_weight(TINY).numpy(), None, intermediate_scales(TINY), workers=1)
    n = TINY.E // world
    sent = np.array([res[r][2]["send_counts"] for r in range(world)])      # [source, destination]
    for r in range(world):
        assert (res[r][0], res[r][1]) == (r * n, n)
        assert res[r][2]["recv_rows"] == int(sent[:, r].sum())
        assert int(((ref["route"].idx >= r * n) & (ref["route"].idx < (r + 1) * n)).sum()) == int(sent[:, r].sum())
        want = ref["out"][r * T_RANK:(r + 1) * T_RANK]
        np.testing.assert_allclose(res[r][3], want, rtol=1e-12, atol=1e-12)


def _rank_main_peer(rank, world, port, accs, out):
    """One gloo rank of the gather exchange with the combine into the owners' memory: the
    accumulators are shared CPU tensors (one per owner, made by the parent), the inter-process
    handle calls are stand-ins that name the owner, and the library's call is replaced by the
    oracle's sums of the rank's experts added into the owners' rows (in rank order, so that the
    stand-in's plain additions do not race)."""
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
        g_h = intermediate_scales(s)
        far = 1 << 40
        log = {"opened": [], "closed": [], "zero_at_start": None}

        def owner_of(addr):
            return rank if addr == accs[rank].data_ptr() else (addr - far) >> 32

        def partial_peer(x_all, w_router, bias, table, rows):
            # every owner zeroed its accumulator before the first collective
            log["zero_at_start"] = all(bool((accs[r] == 0).all()) for r in range(world))
            ref = oracle_layer(s, x_all.float().numpy(), w_router.numpy(), None, g_h, workers=1,
                               expert_range=(layer.e_begin, layer.e_count))["out"]
            for turn in range(world):
                if turn == rank:
                    for t in range(x_all.shape[0]):
                        accs[owner_of(int(table[t // rows]))][t % rows] += torch.from_numpy(ref[t])
                dist.barrier()

        ops = {"alloc": lambda T, H, device: accs[rank],
               "handle": lambda acc: (b"owner %d" % rank, 0),
               "open": lambda h: log["opened"].append(int(h.split()[1])) or far + (int(h.split()[1]) << 32),
               "close": lambda addr: log["closed"].append(addr),
               "partial_peer": partial_peer}
        layer = ExpertParallelLayer(cfg, exchange="peer", peer_ops=ops, finalize=lambda acc: acc.to(torch.bfloat16))
        wr = router_weight(s)
        ys, xs = [], []
        for step in range(2):                       # the second step reuses the mapped table
            accs[rank].fill_(5.0)                   # stale values the step must clear
            x = activations(T_RANK, s, seed=80 + 10 * step + rank)
            ys.append(layer.forward(x, wr).float().numpy())
            xs.append(x.float().numpy())
        layer.close()
        out[rank] = (log["opened"], log["closed"], log["zero_at_start"], ys, xs)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_gloo_ranks_peer_combine_exchange(world):
    """The combine into the owners' memory on gloo ranks: each rank maps every other rank's
    accumulator once, zeroes its own before a collective, the ranks add their experts' sums into
    the owners' rows, and after a second collective every rank's rows are the oracle's whole
    layer on its own tokens, on two consecutive steps; the mappings are released on close."""
    accs = [torch.zeros((T_RANK, 256), dtype=torch.float64).share_memory_() for _ in range(world)]
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main_peer, args=(world, _free_port(), accs, out), nprocs=world, join=True)
        res = dict(out)
    sys.path.insert(0, ROOT)
    from workloads import TINY, router_weight
    from tests.helpers import oracle_layer, intermediate_scales, bf16_half_ulp
    for r in range(world):
        opened, closed, zero_at_start, ys, xs = res[r]
        assert sorted(opened) == [q for q in range(world) if q != r]
        assert len(closed) == world - 1
        assert zero_at_start
    for step in range(2):
        x_all = np.concatenate([res[r][4][step] for r in range(world)])
        ref = oracle_layer(TINY, x_all, router_weight(TINY).numpy(), None, intermediate_scales(TINY), workers=1)
        for r in range(world):
            want = ref["out"][r * T_RANK:(r + 1) * T_RANK]
            got = res[r][3][step]
            assert np.all(np.abs(got - want) <= 2 * bf16_half_ulp(want) + 1e-30)


def test_expert_range_split():
    sys.path.insert(0, ROOT)
    from nvfp4_quantized_moe_group_b200.ep import expert_range
    assert [expert_range(256, r, 8) for r in range(8)] == [(32 * r, 32) for r in range(8)]
    assert expert_range(256, 0, 1) == (0, 256)
    with pytest.raises(ValueError):
        expert_range(256, 0, 3)
