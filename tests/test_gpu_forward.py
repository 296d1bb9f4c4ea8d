"""The whole layer (nvfp4moe_forward) against the oracle: routing (near-tie protocol),
quantised input bit-exact, expert grouping valid and equal to the oracle's, the FP32 SwiGLU
product within the derived bound of the epilogue and its requantisation equal except at near-ties
within that bound, the FP32 output sums within max-abs 2e-2
and relative Frobenius 5e-3, and the BF16 output exactly their round-to-nearest-even."""
import numpy as np
import pytest
import torch

import oracle
import nvfp4_quantized_moe_group_b200 as moe
from workloads import TINY, BEAM, activations, router_weight, expert_weight, zipf_bias
from tests.helpers import (cfg_ns, check_routing, intermediate_scales, oracle_layer, check_output,
                           requant_near_tie)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    moe.lib()


_EXPERTS = {}


def gpu_experts(shape):
    """The layer's experts quantised on the GPU from the seeded BF16 weights (generated on
    the device; the generator is bit-identical to the CPU one)."""
    if shape not in _EXPERTS:
        cfg = moe.make_cfg(shape.E, shape.n_groups, shape.topk_groups, shape.topk, shape.H, shape.I,
                           shape.routed_scale)
        ex = moe.Experts(cfg)
        g_h = intermediate_scales(shape)
        for e in range(shape.E):
            ex.set_from_bf16(e, *(expert_weight(shape, e, w, device="cuda") for w in ("gate", "up", "down")),
                             float(g_h[e]))
        torch.cuda.synchronize()
        _EXPERTS[shape] = ex
    return _EXPERTS[shape]


def check_grouping(dbg, idx, E):
    """The exported grouping is a stable counting sort of the GPU's own routing."""
    counts = dbg["counts"].cpu().numpy()
    offsets = dbg["offsets"].cpu().numpy()
    perm = dbg["perm"].cpu().numpy()
    c, o, p, _ = oracle.permutation(idx, E)
    np.testing.assert_array_equal(counts, c)
    np.testing.assert_array_equal(offsets, o)
    np.testing.assert_array_equal(perm, p)


def run_layer(shape, T, tokens=None, rms_rows=False, bias=None):
    ex = gpu_experts(shape)
    x = activations(T, shape, rms_rows=rms_rows)
    wr = router_weight(shape)
    ws = torch.empty(moe.forward_workspace_bytes(ex.cfg, T), dtype=torch.uint8, device="cuda")
    out, dbg = moe.forward(ex, x.cuda(), wr.cuda(), None if bias is None else bias.cuda(), ws=ws, debug=True,
                           debug_h=True)
    assert moe.status_read(ws) == moe.OK
    g_h = intermediate_scales(shape)
    xn = x.float().numpy()
    bn = None if bias is None else bias.numpy()
    ref = oracle_layer(shape, xn, wr.numpy(), bn, g_h, tokens=tokens)
    r = ref["route"]
    idx = dbg["idx"].cpu().numpy()
    clean, n_flag = check_routing(idx, dbg["w"].cpu().numpy(), r, xn.astype(np.float64),
                                  wr.numpy().astype(np.float64), bn, shape)
    # quantised layer input: bit-exact
    assert np.float32(dbg["g_x"].item()) == ref["g_x"]
    np.testing.assert_array_equal(dbg["xq_codes"].cpu().numpy(), ref["xq_codes"])
    np.testing.assert_array_equal(dbg["xq_scales"].cpu().numpy(), ref["xq_scales"])
    # grouping of the GPU's own routing
    check_grouping(dbg, idx, shape.E)
    if (idx == r.idx).all():
        c, o, p, _ = oracle.permutation(r.idx, shape.E)
        np.testing.assert_array_equal(dbg["perm"].cpu().numpy(), p)
    # requantised intermediate of every checked pair: equal except at near-ties
    perm = dbg["perm"].cpu().numpy()
    pos_of = {int(p): i for i, p in enumerate(perm)}
    hqc = dbg["hq_codes"].cpu().numpy()
    hqs = dbg["hq_scales"].cpu().numpy()
    h_gpu = dbg["h_f32"].cpu().numpy()
    n_el = n_tie = 0
    for (t, j), (h, oc, os_, dh) in ref["inter"].items():
        if idx[t, j] != r.idx[t, j]:
            continue
        e = int(r.idx[t, j])
        i = pos_of[t * shape.topk + j]
        # the FP32 SwiGLU product within the derived bound of the epilogue
        assert np.all(np.abs(h_gpu[i].astype(np.float64) - h) <= dh), f"pair ({t},{j}): h beyond its bound"
        block_tie, elem_tie = requant_near_tie(h, float(g_h[e]), dh)
        sb = hqs[i] != os_
        assert not (sb & ~block_tie).any(), f"pair ({t},{j}): block scale differs away from a near-tie"
        gc = oracle.formats.unpack_codes(hqc[i:i + 1])[0]
        ocu = oracle.formats.unpack_codes(oc[None])[0]
        diff = gc != ocu
        allowed = elem_tie | np.repeat(sb, 16)
        assert not (diff & ~allowed).any(), f"pair ({t},{j}): code differs away from a near-tie"
        n_el += diff.size
        n_tie += int(diff.sum())
    assert n_tie <= max(4, 1e-3 * n_el)
    # outputs of tokens routed identically
    toks = ref["tokens"]
    same = np.array([(idx[t] == r.idx[t]).all() for t in toks])
    assert same.sum() >= 1
    # the FP32 sums within the tolerance; the BF16 output exactly their rounding
    assert torch.equal(out, dbg["acc"].to(torch.bfloat16))
    gpu = dbg["acc"].cpu().numpy()[toks[same]]
    return check_output(gpu, ref["out"][same]), n_flag, n_tie


def test_tiny_layer_all_tokens():
    run_layer(TINY, 64)


def test_tiny_layer_ragged_and_single():
    for T in (1, 5, 130):
        run_layer(TINY, T)


def test_beam_decode_layer():
    run_layer(BEAM, 16, tokens=[0, 5, 11, 15], rms_rows=True)


def test_beam_single_token_layer():
    run_layer(BEAM, 1)


def test_beam_prefill_layer_sampled():
    run_layer(BEAM, 4096, tokens=[0, 1, 2047, 4095])


def test_beam_skewed_layer_sampled():
    run_layer(BEAM, 16384, tokens=[3, 16383], bias=zipf_bias(256))


@pytest.mark.parametrize("T", [16, 64, 65, 200, 600, 4096])
def test_router_logits_within_documented_bound(T):
    """Every FP32 logit the selection used lies within the documented bound of its path: for
    T <= 64 (fused front-end kernel) 32 * 2^-24 * sum|x W| + 2^-24 |logit|; above, the integer
    tensor-core bound 2^-24 |logit| + sum|x - x'| |W| + sum|x| |W - W'| + H 2^(e_x+e_W-28)
    (x', W': the 22- and 30-bit fixed-point rows), which lies well inside the FP32 one."""
    from tests.helpers import router_logit_bound_fp32, router_logit_bound_int
    ex = gpu_experts(BEAM)
    x = activations(T, BEAM, seed=3)
    wr = router_weight(BEAM)
    _, dbg = moe.forward(ex, x.cuda(), wr.cuda(), debug=True)
    torch.cuda.synchronize()
    xn = x.float().numpy().astype(np.float64)
    wn = wr.numpy().astype(np.float64)
    exact = xn @ wn.T
    got = dbg["logits"].cpu().numpy().astype(np.float64)
    err = np.abs(got - exact)
    if T <= 64:
        bound = router_logit_bound_fp32(xn, wn, None, BEAM.H)
        assert np.all(err <= bound), f"max err/bound {np.max(err / bound):.3f}"
        # the bound is not vacuous: errors are a small fraction of it
        assert np.max(err / bound) < 0.5
    else:
        bound = router_logit_bound_int(xn, wn, None, BEAM.H)
        assert np.all(err <= bound), f"max err/bound {np.max(err / bound):.3f}"
        # far tighter than FP32 accumulation: the errors stay a small fraction of the FP32 bound
        b32 = router_logit_bound_fp32(xn, wn, None, BEAM.H)
        rounded = exact.astype(np.float32).astype(np.float64)
        frac = float(np.mean(got == rounded))
        print(f"T={T}: correctly rounded {frac:.4f}, max err/bound {np.max(err / bound):.3g}, "
              f"max err/FP32 bound {np.max(err / b32):.3g}")
        assert np.max(err / b32) < 0.05


def test_integer_router_logits_extreme_rows():
    """The tensor-core logits (T > 64) on rows that stress the fixed-point scaling: a zero row,
    a row whose largest element is 2^40 times the others, a row of subnormal BF16 values, and
    an expert row with the same spread: every logit within the documented integer bound."""
    from tests.helpers import router_logit_bound_int
    ex = gpu_experts(TINY)
    T = 130
    x = activations(T, TINY, seed=9).float()
    x[0] = 0.0
    x[1] = x[1] * 2.0 ** -20
    x[1, 17] = 2.0 ** 20
    x[2] = x[2] * 2.0 ** -130
    x = x.to(torch.bfloat16)
    assert 0 < float(x[2].float().abs().max()) < 2.0 ** -126
    wr = router_weight(TINY).clone()
    wr[5] = wr[5] * 2.0 ** -30
    wr[5, 3] = 1.0e4
    ws = torch.empty(moe.forward_workspace_bytes(ex.cfg, T), dtype=torch.uint8, device="cuda")
    _, dbg = moe.forward(ex, x.cuda(), wr.cuda(), ws=ws, debug=True)
    assert moe.status_read(ws) == moe.OK
    xn = x.float().numpy().astype(np.float64)
    wn = wr.numpy().astype(np.float64)
    exact = xn @ wn.T
    got = dbg["logits"].cpu().numpy().astype(np.float64)
    bound = router_logit_bound_int(xn, wn, None, TINY.H)
    err = np.abs(got - exact)
    assert np.all(err <= bound), f"max err/bound {np.max(err / bound):.3f}"
    assert np.all(got[0] == 0.0)


def test_single_expert_per_token_large_batch():
    """topk = 1 with few experts: the expert segments hold fewer rows than the router's four
    digit planes of the tokens need, so the router takes its own scratch for them; routing
    (near-tie protocol) and outputs still match the oracle."""
    from workloads import LayerShape
    shape = LayerShape(H=256, I=128, E=8, n_groups=2, topk_groups=1, topk=1, routed_scale=1.0,
                       wr_std=1.0 / 16.0, w_std=0.02)
    cfg = moe.make_cfg(shape.E, shape.n_groups, shape.topk_groups, shape.topk, shape.H, shape.I,
                       shape.routed_scale)
    g_h = np.full(shape.E, np.float32(0.004), dtype=np.float32)
    ex = moe.Experts(cfg)
    for e in range(shape.E):
        ex.set_from_bf16(e, *(expert_weight(shape, e, w, device="cuda") for w in ("gate", "up", "down")),
                         float(g_h[e]))
    T = 600
    x = activations(T, shape, seed=13)
    wr = router_weight(shape)
    ws = torch.empty(moe.forward_workspace_bytes(cfg, T), dtype=torch.uint8, device="cuda")
    out, dbg = moe.forward(ex, x.cuda(), wr.cuda(), ws=ws, debug=True)
    assert moe.status_read(ws) == moe.OK
    xn = x.float().numpy()
    toks = [0, 1, 299, 599]
    ref = oracle_layer(shape, xn, wr.numpy(), None, g_h, tokens=toks)
    idx = dbg["idx"].cpu().numpy()
    check_routing(idx, dbg["w"].cpu().numpy(), ref["route"], xn.astype(np.float64),
                  wr.numpy().astype(np.float64), None, shape)
    check_grouping(dbg, idx, shape.E)
    same = np.array([(idx[t] == ref["route"].idx[t]).all() for t in toks])
    assert same.sum() >= 1
    check_output(out.float().cpu().numpy()[np.array(toks)[same]], ref["out"][same], bf16=True)
    ex.close()


@pytest.mark.parametrize("T", [16, 130])
def test_nonfinite_router_weight_reported(T):
    """A NaN in the router weight makes one expert's logits NaN: the forward reports
    NONFINITE, and the selection still holds topk distinct in-range experts per token (the NaN
    expert ranks last), so the grouping and the GEMMs stay inside their buffers."""
    ex = gpu_experts(BEAM)
    x = activations(T, BEAM, seed=5)
    wr = router_weight(BEAM).clone()
    wr[3, 7] = float("nan")
    ws = torch.empty(moe.forward_workspace_bytes(ex.cfg, T), dtype=torch.uint8, device="cuda")
    _, dbg = moe.forward(ex, x.cuda(), wr.cuda(), ws=ws, debug=True)
    assert moe.status_read(ws) == moe.ERR_NONFINITE
    idx = dbg["idx"].cpu().numpy()
    assert ((idx >= 0) & (idx < BEAM.E)).all()
    assert all(len(set(row.tolist())) == BEAM.topk for row in idx)
    assert not (idx == 3).any()
    counts = dbg["counts"].cpu().numpy()
    assert counts.sum() == T * BEAM.topk


def test_front_end_odd_group_layout():
    """The fused front end (T <= 64) with a partial expert tile (E = 48) and groups of 12:
    routing under the near-tie protocol, grouping, and the quantised input bit-exact."""
    from tests.test_gpu_route import ODD_SHAPES
    shape = ODD_SHAPES["gs12"]
    cfg = moe.make_cfg(shape.E, shape.n_groups, shape.topk_groups, shape.topk, shape.H, shape.I,
                       shape.routed_scale)
    ex = moe.Experts(cfg)
    for e in range(shape.E):
        ex.set_from_bf16(e, *(expert_weight(shape, e, w, device="cuda") for w in ("gate", "up", "down")), 1.0)
    for T in (20, 64):
        x = activations(T, shape, seed=11)
        wr = router_weight(shape)
        ws = torch.empty(moe.forward_workspace_bytes(cfg, T), dtype=torch.uint8, device="cuda")
        _, dbg = moe.forward(ex, x.cuda(), wr.cuda(), ws=ws, debug=True)
        assert moe.status_read(ws) == moe.OK
        xn = x.float().numpy()
        r = oracle.route(xn.astype(np.float64), wr.numpy(), cfg_ns(shape), None)
        idx = dbg["idx"].cpu().numpy()
        check_routing(idx, dbg["w"].cpu().numpy(), r, xn.astype(np.float64), wr.numpy().astype(np.float64),
                      None, shape)
        check_grouping(dbg, idx, shape.E)
        xc, xs, gx = oracle.quantize(xn.astype(np.float32))
        assert np.float32(dbg["g_x"].item()) == gx
        np.testing.assert_array_equal(dbg["xq_codes"].cpu().numpy(), xc)
        np.testing.assert_array_equal(dbg["xq_scales"].cpu().numpy(), xs)
    ex.close()


def test_cuda_graph_replay_matches_eager():
    """The whole forward (cooperative front end included) captured in a CUDA graph replays to
    the eager call's routing, grouping and requantised intermediate bit for bit, and to its
    output within one BF16 unit in the last place (the 8 expert outputs of a token are added
    with FP32 atomics, in no fixed order), with a clean status word."""
    ex = gpu_experts(TINY)
    for T in (16, 130):
        x = activations(T, TINY, seed=7).cuda()
        wr = router_weight(TINY).cuda()
        ws = torch.empty(moe.forward_workspace_bytes(ex.cfg, T), dtype=torch.uint8, device="cuda")
        out = torch.empty((T, TINY.H), dtype=torch.bfloat16, device="cuda")
        _, dbg_ref = moe.forward(ex, x, wr, out=out, ws=ws, debug=True)
        torch.cuda.synchronize()
        ref = out.clone()
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.graph(g, stream=s):
            moe.forward(ex, x, wr, out=out, ws=ws)
        out.zero_()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        assert moe.status_read(ws) == moe.OK
        diff = (out.float() - ref.float()).abs()
        assert bool((diff <= 2.0 ** -7 * ref.float().abs() + 1e-30).all())
        # the deterministic intermediates, from one more eager call after the replays
        _, dbg = moe.forward(ex, x, wr, out=out, ws=ws, debug=True)
        for key in ("idx", "w", "perm", "hq_codes", "hq_scales"):
            assert torch.equal(dbg[key], dbg_ref[key]), key
        del g


@pytest.mark.parametrize("shape,T", [(TINY, 16), (TINY, 130), (BEAM, 16), (BEAM, 1100), (BEAM, 4096)])
def test_one_gemm_launch_matches_two(shape, T):
    """The default forward runs both grouped GEMMs in one persistent launch (a down tile waits
    for the gate/up tiles of its rows); nvfp4moe_debug.separate_gemms runs them as two launches.
    Same routing, grouping and requantised intermediate bit for bit, the FP32 sums within the
    reordering of their 8 atomic additions (2^-16 of the row's largest magnitude, which covers
    rows whose terms cancel), clean status words."""
    ex = gpu_experts(shape)
    x = activations(T, shape, seed=41).cuda()
    wr = router_weight(shape).cuda()
    ws = torch.empty(moe.forward_workspace_bytes(ex.cfg, T), dtype=torch.uint8, device="cuda")
    _, d1 = moe.forward(ex, x, wr, ws=ws, debug=True)
    assert moe.status_read(ws) == moe.OK
    _, d2 = moe.forward(ex, x, wr, ws=ws, debug=True, separate_gemms=True)
    assert moe.status_read(ws) == moe.OK
    for key in ("idx", "w", "perm", "hq_codes", "hq_scales"):
        assert torch.equal(d1[key], d2[key]), key
    a1, a2 = d1["acc"].double(), d2["acc"].double()
    tol = 2.0 ** -16 * a2.abs().amax(dim=1, keepdim=True) + 1e-30
    assert bool(((a1 - a2).abs() <= tol).all()), float(((a1 - a2).abs() / tol).max())


def test_experts_set_rejects_misaligned_codes():
    """nvfp4moe_experts_set copies the code rows 16 bytes at a time: a code pointer off a
    16-byte boundary returns NVFP4MOE_ERR_ARG on the host, before anything is enqueued."""
    import ctypes
    from nvfp4_quantized_moe_group_b200._lib import ExpertTensors
    cfg = moe.make_cfg(8, 1, 1, 1, 256, 128, 2.5)
    ex = moe.Experts(cfg)
    buf = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    base = buf.data_ptr()
    assert base % 256 == 0
    for which in (0, 2, 4):                       # gate, up, down codes
        ptrs = [base] * 6
        ptrs[which] = base + 8
        t = ExpertTensors(*ptrs, 1.0, 1.0, 1.0, 1.0)
        assert moe.lib().nvfp4moe_experts_set(ex.handle, 0, ctypes.byref(t), None) == moe.ERR_ARG
        assert moe.last_launch_count() == 0
    torch.cuda.synchronize()
    ex.close()


def test_last_device_status_follows_the_latest_call():
    """nvfp4moe_last_device_status reads the status word of this thread's latest call: clean
    after a clean forward, NONFINITE after a forward whose router weight holds a NaN, while
    the first workspace keeps its own clean word."""
    ex = gpu_experts(BEAM)
    T = 16
    x = activations(T, BEAM, seed=5).cuda()
    wr = router_weight(BEAM).cuda()
    ws = torch.empty(moe.workspace_bytes(ex.cfg, T), dtype=torch.uint8, device="cuda")
    assert ws.numel() == moe.forward_workspace_bytes(ex.cfg, T)
    moe.forward(ex, x, wr, ws=ws)
    assert moe.last_device_status() == moe.OK
    bad = wr.clone()
    bad[3, 7] = float("nan")
    ws2 = torch.empty_like(ws)
    moe.forward(ex, x, bad, ws=ws2)
    assert moe.last_device_status() == moe.ERR_NONFINITE
    assert moe.status_read(ws) == moe.OK and moe.status_read(ws2) == moe.ERR_NONFINITE
