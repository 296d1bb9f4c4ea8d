"""Expert parallelism on one GPU (nvfp4moe_experts_create_local, nvfp4moe_forward_partial,
nvfp4moe_finalize): G ranks are emulated one after another on the same device, with the
all-gather a concatenation and the reduce-scatter an FP32 sum over the ranks' partial sums.
Each rank's FP32 sums are judged against the oracle's sum of that rank's experts'
contributions (max-abs 2e-2, relative Frobenius 5e-3, on tokens the GPU routes as the oracle
does); the ranks' sums must add up to the single-handle layer (up to the order of FP32
additions), a token none of whose experts a rank holds must get an exact zero row from it,
and the rounded result must match nvfp4moe_forward within one BF16 unit."""
import numpy as np
import pytest
import torch

import nvfp4_quantized_moe_group_b200 as moe
from nvfp4_quantized_moe_group_b200.ep import ExpertParallelLayer, expert_range
from workloads import TINY, BEAM, activations, router_weight, expert_weight
import oracle
from tests.helpers import (intermediate_scales, bf16_half_ulp, cfg_ns, oracle_expert_pass, check_output,
                           check_routing)
from tests.test_gpu_forward import gpu_experts

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    moe.lib()


def local_experts(shape, e0, n):
    cfg = moe.make_cfg(shape.E, shape.n_groups, shape.topk_groups, shape.topk, shape.H, shape.I,
                       shape.routed_scale)
    ex = moe.Experts(cfg, e0, n)
    g_h = intermediate_scales(shape)
    for e in range(e0, e0 + n):
        ex.set_from_bf16(e, *(expert_weight(shape, e, w, device="cuda") for w in ("gate", "up", "down")),
                         float(g_h[e]))
    torch.cuda.synchronize()
    return ex


def run_emulated(shape, G, T_rank, seed=50, sample=None):
    """``sample``: gathered token indices whose per-rank sums are compared with the oracle
    (default: all)."""
    full = gpu_experts(shape)
    xs_cpu = [activations(T_rank, shape, seed=seed + r) for r in range(G)]
    x_all_cpu = torch.cat(xs_cpu)
    x_all = x_all_cpu.cuda()
    wr_cpu = router_weight(shape)
    wr = wr_cpu.cuda()
    g_h = intermediate_scales(shape)
    sample = np.arange(G * T_rank) if sample is None else np.asarray(sample)
    acc_full, dbg = moe.forward_partial(full, x_all, wr, debug=True)
    out_full = moe.forward(full, x_all, wr)
    idx = dbg["idx"].cpu().numpy()
    # the oracle: routing of all gathered tokens, every sampled pair's expert evaluated once
    xn = x_all_cpu.float().numpy()
    r_or = oracle.route(xn.astype(np.float64), wr_cpu.numpy().astype(np.float64), cfg_ns(shape), None)
    xc, xsc, gx = oracle.quantize(xn)
    same = (idx[sample] == r_or.idx[sample]).all(axis=1)
    assert same.mean() > 0.9
    checked = sample[same]
    rows = {}
    for i, t in enumerate(checked):
        for j in range(shape.topk):
            rows.setdefault(int(r_or.idx[t, j]), []).append((i, int(t), j))
    xhat = oracle.dequantize(xc[checked], xsc[checked], gx)
    ys = oracle_expert_pass(shape, {e: (xhat[[i for i, _, _ in v]], float(g_h[e]), None, None)
                                    for e, v in rows.items()})
    accs = []
    for r in range(G):
        e0, n = expert_range(shape.E, r, G)
        ex = local_experts(shape, e0, n)
        assert (ex.e_begin, ex.e_count) == (e0, n)
        acc_r, dbg_r = moe.forward_partial(ex, x_all, wr, debug=True)
        # every rank routes the gathered tokens identically
        np.testing.assert_array_equal(dbg_r["idx"].cpu().numpy(), idx, err_msg=f"rank {r} routes differently")
        # tokens with no selected expert in the rank's range get an exact zero row
        none_local = ~((idx >= e0) & (idx < e0 + n)).any(axis=1)
        a = acc_r.cpu().numpy()
        assert np.all(a[none_local] == 0.0), f"rank {r}: non-zero rows for tokens without a local expert"
        assert not np.any(np.all(a[~none_local] == 0.0, axis=1)), f"rank {r}: a token's local experts added nothing"
        # the rank's sums against the oracle's sum over the rank's experts
        ref = np.zeros((len(checked), shape.H))
        for e, v in rows.items():
            if e0 <= e < e0 + n:
                for m, (i, t, j) in enumerate(v):
                    ref[i] += r_or.w[t, j] * ys[e][0][m]
        check_output(a[checked], ref)
        accs.append(acc_r)
        ex.close()
    total = accs[0].clone()
    for acc_r in accs[1:]:
        total += acc_r
    af = acc_full.cpu().numpy()
    diff = np.abs(total.cpu().numpy() - af)
    # both are FP32 sums of the same 8 weighted expert rows per token in different orders:
    # they differ by FP32 roundings, a few units of 2^-24 of the row's magnitudes (a missing
    # or doubled expert row would differ by a whole contribution)
    row_scale = np.abs(af).max(axis=1, keepdims=True)
    lim = 2.0 ** -16 * row_scale + 1e-30
    assert np.all(diff <= lim), f"max diff/row scale {np.max(diff / (row_scale + 1e-30)):.3g}"
    # each rank's own rows after the reduce-scatter, rounded: the single-GPU layer to one BF16
    # unit, except where the FP32 difference straddles a BF16 rounding boundary
    out_ep = moe.finalize(total).float().cpu().numpy()
    of = out_full.float().cpu().numpy()
    bad = np.abs(out_ep - of) > 2 * bf16_half_ulp(of) + 1e-30
    assert bad.sum() <= max(4, 1e-4 * bad.size), f"{int(bad.sum())} outputs beyond one BF16 unit"
    return out_ep


@pytest.mark.parametrize("G,T_rank", [(2, 24), (4, 24), (8, 8)])
def test_tiny_emulated_ranks(G, T_rank):
    run_emulated(TINY, G, T_rank)


def test_beam_decode_eight_ranks():
    """Beam decode on 8 emulated ranks: 16 tokens each, 128 gathered tokens."""
    run_emulated(BEAM, 8, 16, sample=[0, 21, 47, 70, 101, 127])


def run_peer_emulated(shape, G, T_rank, seed=90):
    """The combine into the owners' memory (nvfp4moe_forward_partial_peer), G ranks emulated one
    after another on one GPU: every rank's call adds its experts' weighted rows into the G
    owners' accumulators (here all on this device, their addresses in one table).  The owners'
    sums must equal the single-handle layer's FP32 sums up to the order of FP32 additions (the
    gather emulation above checks each rank's share against the oracle), each owner must get
    exactly its own tokens' rows, and the rounded rows must match nvfp4moe_forward within one
    BF16 unit."""
    full = gpu_experts(shape)
    x_all = torch.cat([activations(T_rank, shape, seed=seed + r) for r in range(G)]).cuda()
    wr = router_weight(shape).cuda()
    acc_full = moe.forward_partial(full, x_all, wr)
    out_full = moe.forward(full, x_all, wr)
    # owners' accumulators with a canary row after each: nothing may land outside the owners' rows
    store = torch.zeros((G, T_rank + 1, shape.H), dtype=torch.float32, device="cuda")
    store[:, T_rank] = 7.0
    table = torch.tensor([store[r].data_ptr() for r in range(G)], dtype=torch.int64, device="cuda")
    for r in range(G):
        e0, n = expert_range(shape.E, r, G)
        ex = local_experts(shape, e0, n)
        moe.forward_partial_peer(ex, x_all, wr, None, table, T_rank)
        torch.cuda.synchronize()
        ex.close()
    assert bool((store[:, T_rank] == 7.0).all()), "a row outside the owners' token rows was written"
    total = store[:, :T_rank].reshape(G * T_rank, shape.H).cpu().numpy()
    af = acc_full.cpu().numpy()
    row_scale = np.abs(af).max(axis=1, keepdims=True)
    diff = np.abs(total - af)
    assert np.all(diff <= 2.0 ** -16 * row_scale + 1e-30), f"max diff/row scale {np.max(diff / (row_scale + 1e-30)):.3g}"
    out = torch.cat([moe.finalize(store[r, :T_rank].contiguous()) for r in range(G)]).float().cpu().numpy()
    of = out_full.float().cpu().numpy()
    bad = np.abs(out - of) > 2 * bf16_half_ulp(of) + 1e-30
    assert bad.sum() <= max(4, 1e-4 * bad.size), f"{int(bad.sum())} outputs beyond one BF16 unit"


@pytest.mark.parametrize("G,T_rank", [(2, 24), (4, 40)])
def test_tiny_peer_combine_emulated(G, T_rank):
    run_peer_emulated(TINY, G, T_rank)


def test_beam_peer_combine_emulated():
    """Beam on 4 emulated ranks with 300 tokens each: full segments (two GEMM launches, the
    staged bulk reductions) into the owners' accumulators."""
    run_peer_emulated(BEAM, 4, 300)


def test_beam_peer_combine_decode_emulated():
    """Beam decode on 8 emulated ranks with 16 tokens each: the one-launch GEMMs' register
    reductions into the owners' accumulators."""
    run_peer_emulated(BEAM, 8, 16)


def test_single_rank_peer_exchange_matches_forward():
    """ExpertParallelLayer(exchange="peer") without a process group: its own accumulator is the
    only owner; the result is the whole layer."""
    cfg = moe.make_cfg(TINY.E, TINY.n_groups, TINY.topk_groups, TINY.topk, TINY.H, TINY.I, TINY.routed_scale)
    layer = ExpertParallelLayer(cfg, exchange="peer")
    ex = layer.create_experts()
    g_h = intermediate_scales(TINY)
    for e in range(TINY.E):
        ex.set_from_bf16(e, *(expert_weight(TINY, e, w, device="cuda") for w in ("gate", "up", "down")),
                         float(g_h[e]))
    x = activations(40, TINY, seed=9).cuda()
    wr = router_weight(TINY).cuda()
    want = moe.forward(gpu_experts(TINY), x, wr).float().cpu().numpy()
    for _ in range(2):                          # the second step reuses the table and re-zeroes
        got = layer.forward(x, wr).float().cpu().numpy()
        assert np.all(np.abs(got - want) <= 2 * bf16_half_ulp(want) + 1e-30)
    layer.close()


def test_local_handle_rejects_foreign_experts_and_bad_ranges():
    cfg = moe.make_cfg(TINY.E, TINY.n_groups, TINY.topk_groups, TINY.topk, TINY.H, TINY.I, TINY.routed_scale)
    ex = moe.Experts(cfg, 8, 8)
    w = [expert_weight(TINY, 3, n, device="cuda") for n in ("gate", "up", "down")]
    with pytest.raises(moe.NvFp4MoeError):
        ex.set_from_bf16(3, *w, 1.0)                    # expert 3 is not in 8 .. 15
    ex.close()
    for e0, n in ((-1, 4), (30, 4), (0, 0)):
        with pytest.raises(moe.NvFp4MoeError):
            moe.Experts(cfg, e0, n)


def test_single_rank_layer_matches_forward():
    """ExpertParallelLayer without a process group: the whole layer on this GPU."""
    cfg = moe.make_cfg(TINY.E, TINY.n_groups, TINY.topk_groups, TINY.topk, TINY.H, TINY.I, TINY.routed_scale)
    layer = ExpertParallelLayer(cfg)
    assert (layer.world, layer.e_begin, layer.e_count) == (1, 0, TINY.E)
    ex = layer.create_experts()
    g_h = intermediate_scales(TINY)
    for e in range(TINY.E):
        ex.set_from_bf16(e, *(expert_weight(TINY, e, w, device="cuda") for w in ("gate", "up", "down")),
                         float(g_h[e]))
    x = activations(40, TINY, seed=7).cuda()
    wr = router_weight(TINY).cuda()
    got = layer.forward(x, wr).float().cpu().numpy()
    want = moe.forward(gpu_experts(TINY), x, wr).float().cpu().numpy()
    assert np.all(np.abs(got - want) <= 2 * bf16_half_ulp(want) + 1e-30)
    layer.close()


def run_all_to_all_emulated(shape, G, T_rank, seed=70, sample=None):
    """The all-to-all exchange (nvfp4moe_amax, _ep_dispatch, _ep_experts, _ep_combine) with G ranks
    emulated one after another on this GPU, each collective a host-side concatenation of the
    ranks' buffers.  Checked: every rank's dispatched rows are the oracle's quantisation of its
    tokens with the global scale of all ranks' tokens, in the oracle's expert-major order, with
    the oracle's per-rank counts (bit-exact, where the GPU routes as the oracle does); every
    rank's output equals nvfp4moe_forward on the concatenated batch up to the order of the FP32
    additions; the sampled tokens' FP32 sums are within the layer tolerance of the oracle, and
    the BF16 output is their exact rounding."""
    cfg = moe.make_cfg(shape.E, shape.n_groups, shape.topk_groups, shape.topk, shape.H, shape.I, shape.routed_scale)
    k, H = shape.topk, shape.H
    xs_cpu = [activations(T_rank, shape, seed=seed + r) for r in range(G)]
    xs = [x.cuda() for x in xs_cpu]
    wr_cpu = router_weight(shape)
    wr = wr_cpu.cuda()
    g_h = intermediate_scales(shape)
    # 1. the global amax
    amax = torch.stack([moe.amax(x) for x in xs]).max(dim=0).values
    x_all_cpu = torch.cat(xs_cpu)
    ref_bits = int((x_all_cpu.view(torch.int16).to(torch.int32) & 0x7FFF).max())
    assert int(amax.item()) == ref_bits
    # 2. dispatch on every rank
    sends = [moe.ep_dispatch(cfg, G, x, wr, None, amax) for x in xs]
    torch.cuda.synchronize()
    g_glob = oracle.global_scale(np.array([ref_bits << 16], dtype=np.uint32).view(np.float32)[0])
    epr = shape.E // G
    idx_gpu = []
    for r, sd in enumerate(sends):
        xn = xs_cpu[r].float().numpy()
        ro = oracle.route(xn.astype(np.float64), wr_cpu.numpy().astype(np.float64), cfg_ns(shape), None)
        # the rank's routing (the kernels nvfp4moe_route runs) under the near-tie protocol; the
        # layout is then fixed by it
        gi, gw = moe.route(cfg, xs[r], wr)
        gi, gw = gi.cpu().numpy(), gw.cpu().numpy()
        check_routing(gi, gw, ro, xn.astype(np.float64), wr_cpu.numpy().astype(np.float64), None, shape)
        idx_gpu.append(gi)
        codes, scales, _ = oracle.quantize(xn, g=g_glob)
        counts, _, perm, inv = oracle.permutation(gi, shape.E)
        np.testing.assert_array_equal(sd["rank_counts"].cpu().numpy(), counts.reshape(G, epr).sum(axis=1))
        np.testing.assert_array_equal(sd["codes"].cpu().numpy(), codes[perm // k])
        np.testing.assert_array_equal(sd["scales"].cpu().numpy(), scales[perm // k])
        np.testing.assert_array_equal(sd["expert"].cpu().numpy(), gi.reshape(-1)[perm] % epr)
        np.testing.assert_array_equal(sd["pos"].cpu().numpy(), inv.reshape(-1))
        np.testing.assert_array_equal(sd["w"].cpu().numpy(), gw.reshape(-1)[perm])
    # 3. rows to their experts' ranks
    counts = [sd["rank_counts"].cpu().tolist() for sd in sends]
    offs = [np.concatenate([[0], np.cumsum(c)]) for c in counts]
    rows_back = [[None] * G for _ in range(G)]
    for d in range(G):
        recv = {key: torch.cat([sends[src][key][offs[src][d]:offs[src][d + 1]] for src in range(G)])
                for key in ("codes", "scales", "expert", "w")}
        ex = local_experts(shape, d * epr, epr)
        rows = moe.ep_experts(ex, recv["codes"], recv["scales"], recv["expert"], recv["w"], amax)
        torch.cuda.synchronize()
        ex.close()
        o = 0
        for src in range(G):
            n = counts[src][d]
            rows_back[src][d] = rows[o:o + n]
            o += n
    # 4. rows back and the combine
    outs, accs = [], []
    for src in range(G):
        back = torch.cat(rows_back[src])
        out = moe.ep_combine(back, sends[src]["pos"], T_rank, k)
        b = back.cpu().numpy()
        p = sends[src]["pos"].cpu().numpy().reshape(T_rank, k)
        acc = np.zeros((T_rank, H), dtype=np.float32)
        for j in range(k):
            acc = (acc + b[p[:, j]]).astype(np.float32)
        assert torch.equal(out.cpu(), torch.from_numpy(acc).to(torch.bfloat16)), "combine is not the slot-order sum"
        outs.append(out.float().cpu().numpy())
        accs.append(acc)
    # the single-GPU layer on the concatenated batch, same routing and codes
    full = gpu_experts(shape)
    single = moe.forward(full, torch.cat(xs), wr).float().cpu().numpy()
    got = np.concatenate(outs)
    row = np.abs(single).max(axis=1, keepdims=True)
    assert np.all(np.abs(got - single) <= 2 * bf16_half_ulp(single) + 2.0 ** -16 * row + 1e-30)
    # sampled tokens against the oracle (FP32 sums)
    acc_all = np.concatenate(accs)
    T_all = G * T_rank
    sample = np.arange(T_all) if sample is None else np.asarray(sample)
    xn = x_all_cpu.float().numpy()
    r_or = oracle.route(xn.astype(np.float64), wr_cpu.numpy().astype(np.float64), cfg_ns(shape), None)
    xc, xsc, gx = oracle.quantize(xn)
    assert gx == g_glob
    same = (np.concatenate(idx_gpu)[sample] == r_or.idx[sample]).all(axis=1)
    assert same.mean() > 0.9
    sample = sample[same]
    need = {}
    for i, t in enumerate(sample):
        for j in range(k):
            need.setdefault(int(r_or.idx[t, j]), []).append((i, int(t), j))
    xhat = oracle.dequantize(xc[sample], xsc[sample], gx)
    ys = oracle_expert_pass(shape, {e: (xhat[[i for i, _, _ in v]], float(g_h[e]), None, None) for e, v in need.items()})
    ref = np.zeros((len(sample), H))
    for e, v in need.items():
        for m, (i, t, j) in enumerate(v):
            ref[i] += r_or.w[t, j] * ys[e][0][m]
    check_output(acc_all[sample], ref)


@pytest.mark.parametrize("G,T_rank", [(2, 24), (4, 40)])
def test_tiny_all_to_all_emulated(G, T_rank):
    run_all_to_all_emulated(TINY, G, T_rank)


def test_beam_all_to_all_eight_ranks_full_segments():
    """Beam prefill on 8 emulated ranks of 512 tokens: every receiving rank groups about 4096
    rows over its 32 experts (the full-segment GEMM epilogues)."""
    run_all_to_all_emulated(BEAM, 8, 512, sample=[0, 700, 1500, 2222, 3000, 4095])


def test_ep_experts_checks_received_expert_indices_on_the_device():
    """Expert indices arrive from other ranks: one outside the handle's experts is replaced on
    the device (every access stays in bounds) and reported as NVFP4MOE_ERR_ARG."""
    shape = TINY
    cfg = moe.make_cfg(shape.E, shape.n_groups, shape.topk_groups, shape.topk, shape.H, shape.I, shape.routed_scale)
    ex = local_experts(shape, 0, 16)
    x = activations(4, shape, seed=90).cuda()
    amax = moe.amax(x)
    codes, scales, _ = moe.quantize(x)
    w = torch.ones(4, dtype=torch.float32, device="cuda")
    good = torch.tensor([3, 0, 15, 5], dtype=torch.int32, device="cuda")
    rows = moe.ep_experts(ex, codes, scales, good, w, amax)
    assert moe.last_device_status() == moe.OK
    bad = torch.tensor([3, -1, 16, 5], dtype=torch.int32, device="cuda")
    rows_bad = moe.ep_experts(ex, codes, scales, bad, w, amax)
    assert moe.last_device_status() == moe.ERR_ARG
    assert bool(torch.isfinite(rows_bad).all())
    # the rows with valid indices are unchanged by the bad ones
    for i in (0, 3):
        assert torch.equal(rows_bad[i], rows[i])
    ex.close()


def test_ep_experts_and_combine_with_nothing_to_do():
    """A rank that receives no row (every pair routed elsewhere) runs nvfp4moe_ep_experts on zero
    rows: status clean, nothing written; a combine of zero tokens enqueues nothing."""
    shape = TINY
    ex = local_experts(shape, 16, 16)
    amax = moe.amax(activations(4, shape, seed=91).cuda())
    empty_codes = torch.empty((0, shape.H // 2), dtype=torch.uint8, device="cuda")
    empty_scales = torch.empty((0, shape.H // 16), dtype=torch.uint8, device="cuda")
    rows = moe.ep_experts(ex, empty_codes, empty_scales, torch.empty(0, dtype=torch.int32, device="cuda"),
                          torch.empty(0, dtype=torch.float32, device="cuda"), amax)
    assert tuple(rows.shape) == (0, shape.H)
    assert moe.last_device_status() == moe.OK
    out = moe.ep_combine(torch.empty((0, shape.H), dtype=torch.float32, device="cuda"),
                         torch.empty(0, dtype=torch.int32, device="cuda"), 0, shape.topk)
    assert tuple(out.shape) == (0, shape.H)
    ex.close()
