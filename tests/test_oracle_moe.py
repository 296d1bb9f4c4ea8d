"""Pins for the oracle's expert grouping, SwiGLU expert MLP and layer combine (CPU only)."""
import math
import types

import numpy as np
import torch

import oracle
from oracle.moe import QuantTensor, _bf16_round
from workloads import TINY, activations, router_weight, expert_weight


def _cfg(shape):
    return types.SimpleNamespace(E=shape.E, n_groups=shape.n_groups, topk_groups=shape.topk_groups,
                                 topk=shape.topk, routed_scale=shape.routed_scale)


def test_permutation_against_loop_and_invariants():
    rng = np.random.default_rng(0)
    T, k, E = 37, 8, 32
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)])
    counts, offsets, perm, inv = oracle.permutation(idx, E)
    # plain loop: walk experts, then tokens in order
    want = [t * k + j for e in range(E) for t in range(T) for j in range(k) if idx[t, j] == e]
    assert perm.tolist() == want
    assert counts.sum() == T * k and offsets[-1] == T * k
    np.testing.assert_array_equal(np.diff(offsets), counts)
    np.testing.assert_array_equal(perm[inv.reshape(-1)], np.arange(T * k))
    for e in range(E):
        seg = perm[offsets[e]:offsets[e + 1]]
        assert np.all(idx.reshape(-1)[seg] == e) and np.all(np.diff(seg // k) > 0)


def test_permutation_empty_experts():
    idx = np.array([[3, 1], [3, 1]])
    counts, offsets, perm, inv = oracle.permutation(idx, 6)
    assert counts.tolist() == [0, 2, 0, 2, 0, 0]
    assert offsets.tolist() == [0, 0, 2, 2, 4, 4, 4]
    assert perm.tolist() == [1, 3, 0, 2]


def _qt(w):
    return oracle.quantize_tensor(w.float().numpy())


def test_expert_mlp_one_hot_input_closed_form():
    """x = v * e_k picks column k of the gate/up weights: h_i = silu(v Wg[i,k]) * v Wu[i,k]."""
    H, I = 64, 32
    gate = _qt(expert_weight(TINY, 0, "gate")[:I, :H] * 40)
    up = _qt(expert_weight(TINY, 0, "up")[:I, :H] * 40)
    down = _qt(expert_weight(TINY, 0, "down")[:H, :I] * 40)
    v, k = 1.5, 11
    x = np.zeros((1, H))
    x[0, k] = v
    res = oracle.expert_mlp(x, gate, up, down, np.float32(0.01))
    wg = gate.dequant()[:, k]
    wu = up.dequant()[:, k]
    h = (v * wg) / (1 + np.exp(-v * wg)) * (v * wu)
    np.testing.assert_allclose(res["h"][0], h, rtol=1e-14, atol=1e-300)
    # y = dequant(requant(h)) @ Wd^T, written as a per-output loop
    hh = oracle.dequantize(res["hq_codes"], res["hq_scales"], np.float32(0.01))[0]
    wd = down.dequant()
    y = np.array([sum(hh[i] * wd[n, i] for i in range(I)) for n in range(H)])
    np.testing.assert_allclose(res["y"][0], y, rtol=1e-12, atol=1e-15)


def test_swiglu_special_values():
    H, I = 32, 16
    zero = QuantTensor(np.zeros((I, H // 2), np.uint8), np.zeros((I, H // 16), np.uint8), np.float32(1))
    up = _qt(expert_weight(TINY, 1, "up")[:I, :H])
    down = _qt(expert_weight(TINY, 1, "down")[:H, :I])
    res = oracle.expert_mlp(np.ones((2, H)), zero, up, down, np.float32(0.01))
    assert np.all(res["h"] == 0) and np.all(res["y"] == 0)


def _tiny_layer(T=24):
    shape = TINY
    x = activations(T, shape).float().numpy()
    wr = router_weight(shape).numpy()
    ex = {e: tuple(_qt(expert_weight(shape, e, w)) for w in ("gate", "up", "down")) for e in range(shape.E)}
    # a different static scale per expert, so that an expert's h quantised with another
    # expert's scale shows
    g_h = (np.float32(0.002) * (1 + np.arange(shape.E, dtype=np.float32) / shape.E)).astype(np.float32)
    return shape, x, wr, ex, g_h


def test_layer_combine_matches_dense_formulation():
    """Gathered per-expert evaluation == every expert on every token, then a dense [T, E]
    weight matrix; pins the pair/slot/expert indexing of the combine."""
    shape, x, wr, ex, g_h = _tiny_layer()
    cfg = _cfg(shape)
    res = oracle.moe_forward(x, wr, cfg, lambda e: ex[e], g_h)
    r = res["route"]
    xhat = oracle.dequantize(res["xq_codes"], res["xq_scales"], res["g_x"])
    dense_w = np.zeros((x.shape[0], shape.E))
    np.put_along_axis(dense_w, r.idx, r.w, axis=1)
    y_all = np.stack([oracle.expert_mlp(xhat, *ex[e], g_h[e])["y"] for e in range(shape.E)], axis=1)
    out = np.einsum("te,teh->th", dense_w, y_all)
    np.testing.assert_allclose(res["out"], out, rtol=1e-12, atol=1e-12)


def test_layer_sampled_tokens_equal_full_run():
    shape, x, wr, ex, g_h = _tiny_layer()
    cfg = _cfg(shape)
    full = oracle.moe_forward(x, wr, cfg, lambda e: ex[e], g_h)
    part = oracle.moe_forward(x, wr, cfg, lambda e: ex[e], g_h, tokens=[3, 17, 5])
    np.testing.assert_allclose(part["out"], full["out"][[3, 17, 5]], rtol=1e-12, atol=1e-15)


def test_single_expert_layer_is_scaled_expert():
    shape, x, wr, ex, g_h = _tiny_layer(8)
    cfg = types.SimpleNamespace(E=shape.E, n_groups=1, topk_groups=1, topk=1, routed_scale=2.5)
    res = oracle.moe_forward(x, wr, cfg, lambda e: ex[e], g_h)
    xhat = oracle.dequantize(res["xq_codes"], res["xq_scales"], res["g_x"])
    for t in range(8):
        e = res["route"].idx[t, 0]
        y = oracle.expert_mlp(xhat[t:t + 1], *ex[e], g_h[e])["y"][0]
        np.testing.assert_allclose(res["out"][t], 2.5 * y, rtol=1e-12, atol=1e-15)


def test_bf16_rounding_matches_torch():
    v = np.random.default_rng(0).standard_normal(100000) * 3
    ref = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    # torch rounds FP64 -> BF16 via FP32; away from double-rounding cases they agree
    v32 = v.astype(np.float32).astype(np.float64)
    np.testing.assert_array_equal(_bf16_round(v32), torch.from_numpy(v32).to(torch.bfloat16).double().numpy())
    assert np.mean(_bf16_round(v) == ref) > 0.999


def test_worked_layer_example():
    """A whole layer worked by hand, with operands NVFP4 represents exactly.

    Layer: E = 4 experts in 2 groups of 2, keep 1 group, top 2, routed scale 2.5; H = 32,
    I = 16.  One token, x[3] = 2.625 and zeros elsewhere.

    * Input quantisation: A = 2.625, g = 2.625 / 2688 = 2^-10; block 0 scales 2.625 * r_t to
      448 (code 126), d = 0.4375, 2.625 / d = 6 -> code 7 (byte 1 = 0x70); block 1 is zero
      (scale 0).  So xhat[3] = 2.625 exactly.
    * Router (on the BF16 x): W[:, 3] = [1, -0.5, 0.25, 0.75], logits
      l = [2.625, -1.3125, 0.65625, 1.96875].  Group sums: g0 = s(2.625) + s(-1.3125) = 1.144,
      g1 = s(0.65625) + s(1.96875) = 1.536, so group 1 is kept and the experts are 3, 2 (score
      order), although expert 0 has the best single score; w = 2.5 s / (s2 + s3).
    * Experts, the same gate and up for all: gate[5, 3] = 21 = 2688 * 2^-7 and
      up[5, 3] = 0.328125 = 2688 * 2^-13, each the maximum of its tensor, so g = 2^-7 and 2^-13,
      block scale 448, code 6 and the values decode exactly.  gate = 2.625 * 21 = 55.125,
      up = 2.625 * 0.328125 = 0.861328125, silu(55.125) = 55.125 in FP64 (e^-55 is below half
      an ulp), h[5] = 194481 / 4096 = 47.480712890625 (exact in FP32).
    * Requantisation of h with g_h = 1/8: r_t = fp32(1 / 0.75), h * r_t = 63.31 -> nearest E4M3
      64 (code 104), d = 8, h / d = 5.94 -> E2M1 6 (code 7, byte 2 = 0x70): hhat[5] = 48.
    * Down: expert e has down[9, 5] = 21 * 2^e (g = 2^(e-7), exact), y_e[9] = 48 * 21 * 2^e.
    * Combine: out[9] = 1008 (8 w_3 + 4 w_2) = 15838.84..., every other output 0; BF16 (a step
      of 64 there): 15808."""
    H, I, E = 32, 16, 4
    cfg = types.SimpleNamespace(E=E, n_groups=2, topk_groups=1, topk=2, routed_scale=2.5)
    x = np.zeros((1, H), np.float32)
    x[0, 3] = 2.625
    wr = np.zeros((E, H), np.float32)
    wr[:, 3] = [1.0, -0.5, 0.25, 0.75]
    gate = np.zeros((I, H), np.float32)
    gate[5, 3] = 21.0
    up = np.zeros((I, H), np.float32)
    up[5, 3] = 0.328125
    ex = {}
    for e in range(E):
        down = np.zeros((H, I), np.float32)
        down[9, 5] = 21.0 * 2 ** e
        ex[e] = (oracle.quantize_tensor(gate), oracle.quantize_tensor(up), oracle.quantize_tensor(down))
    res = oracle.moe_forward(x, wr, cfg, lambda e: ex[e], np.full(E, 0.125, np.float32), keep_intermediates=True)

    assert res["g_x"] == np.float32(2.0 ** -10)
    want_xq = np.zeros((1, H // 2), np.uint8)
    want_xq[0, 1] = 0x70
    np.testing.assert_array_equal(res["xq_codes"], want_xq)
    np.testing.assert_array_equal(res["xq_scales"], [[126, 0]])
    r = res["route"]
    assert list(r.groups[0]) == [1] and list(r.idx[0]) == [3, 2]
    l = [2.625, -1.3125, 0.65625, 1.96875]
    s = [1.0 / (1.0 + math.exp(-v)) for v in l]
    w3, w2 = 2.5 * s[3] / (s[2] + s[3]), 2.5 * s[2] / (s[2] + s[3])
    np.testing.assert_allclose(r.w[0], [w3, w2], rtol=1e-15)
    for j in (0, 1):
        it = res["inter"][(0, j)]
        assert it["gate"][5] == 55.125 and it["up"][5] == 0.861328125
        assert it["h"][5] == 194481 / 4096 and np.count_nonzero(it["h"]) == 1
        np.testing.assert_array_equal(it["hq_scales"], [104])
        assert it["hq_codes"][2] == 0x70 and np.count_nonzero(it["hq_codes"]) == 1
    out = res["out"][0]
    assert np.flatnonzero(out).tolist() == [9]
    np.testing.assert_allclose(out[9], 1008 * (8 * w3 + 4 * w2), rtol=1e-14)
    assert res["out_bf16"][0, 9] == 15808.0


def test_stored_intermediate_scales_are_reproducible():
    """The stored static scales g_h of the tiny layer are what the committed calibration
    script computes from the oracle today."""
    import importlib.util
    import os
    from tests.helpers import intermediate_scales
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    spec = importlib.util.spec_from_file_location(
        "make_intermediate_scales", os.path.join(root, "tests", "golden", "make_intermediate_scales.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    np.testing.assert_array_equal(mod.calibrate(TINY), intermediate_scales(TINY))
