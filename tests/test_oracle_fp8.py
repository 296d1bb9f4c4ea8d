"""Pins of oracle/fp8.py (the FP8 W8A8 variant of "FP8 quantization", sections "Quantization
scheme" and "Quantization method"): the row maximum maps to +-448, the rounding error bound,
sign symmetry, zero rows, idempotence, PyTorch's float8_e4m3fn cast, and a closed-form
expert MLP."""
import numpy as np
import torch

import oracle
from oracle import fp8


def _rows(seed, rows=6, cols=48, scale=1.0):
    rng = np.random.default_rng(seed)
    v = rng.standard_normal((rows, cols)) * scale * np.exp(rng.standard_normal((rows, 1)))
    return oracle.moe._bf16_round(v).astype(np.float32)


def test_row_maximum_maps_to_448():
    v = _rows(0)
    codes, s = fp8.quantize_rows(v)
    j = np.argmax(np.abs(v), axis=1)
    c = codes[np.arange(v.shape[0]), j]
    assert np.all((c & 0x7F) == 0x7E)
    assert np.all((c >> 7) == (v[np.arange(v.shape[0]), j] < 0))


def test_rounding_error_bound_and_library_cast():
    v = _rows(1, rows=8, cols=256)
    codes, s = fp8.quantize_rows(v)
    q = (v / s[:, None]).astype(np.float32)
    # PyTorch's E4M3 cast (round to nearest even) of the same FP32 quotients
    ref = torch.from_numpy(q).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(codes, ref)
    deq = fp8.dequantize_rows(codes, s)
    err = np.abs(deq - v.astype(np.float64))
    # 3 mantissa bits: half a step is 2^-4 relative for normals, 2^-10 s absolute below 2^-6 s
    assert np.all(err <= np.maximum(np.abs(v) * 2.0 ** -4, 2.0 ** -10 * s[:, None]) * (1 + 1e-6))


def test_sign_symmetry_zero_rows_idempotence():
    v = _rows(2)
    c1, s1 = fp8.quantize_rows(v)
    c2, s2 = fp8.quantize_rows(-v)
    np.testing.assert_array_equal(s1, s2)
    nz = v != 0
    np.testing.assert_array_equal(c2[nz], c1[nz] ^ 0x80)
    z = np.zeros((2, 32), dtype=np.float32)
    cz, sz = fp8.quantize_rows(z)
    assert np.all(cz == 0) and np.all(sz == 1.0)
    deq = fp8.dequantize_rows(c1, s1).astype(np.float32)
    c3, s3 = fp8.quantize_rows(deq)
    np.testing.assert_array_equal(s3, s1)
    np.testing.assert_array_equal(c3, c1)


def test_expert_mlp_closed_form():
    """Operands FP8 represents exactly with exact per-row scales (row maxima 448 and 896 give
    s = 1 and 2): x = [1/256, 3/256], gate = 448 I, up = 896 I, down = 448 I."""
    eye = np.eye(2, dtype=np.float32)
    gate, up, down = fp8.Fp8Tensor(448 * eye), fp8.Fp8Tensor(896 * eye), fp8.Fp8Tensor(448 * eye)
    assert list(gate.scales) == [1.0, 1.0] and list(up.scales) == [2.0, 2.0]
    xhat = np.array([[1 / 256, 3 / 256]])
    res = fp8.expert_mlp_fp8(xhat, gate, up, down)
    g, u = 448 * xhat[0], 896 * xhat[0]
    h = (g / (1 + np.exp(-g)) * u).astype(np.float32)
    np.testing.assert_array_equal(res["h"][0], h)
    hq = fp8.dequantize_rows(*fp8.quantize_rows(h[None]))[0]
    np.testing.assert_allclose(res["y"][0], 448 * hq, rtol=1e-15)


def test_division_reading_at_an_e4m3_tie():
    """The reading "code = E4M3_rne(fp32(v / s)) with one IEEE division" at a value where it
    matters: for the row [1.078125, 0.01263427734375] the scale is s = fp32(1.078125 / 448) and
    fp32(v / s) is exactly 5.25, the midpoint of E4M3 5.0 (code 0x4A) and 5.5 (0x4B), so the
    tie goes to the even code 0x4A; multiplying by fp32(1 / s) instead lands one FP32 step above
    the midpoint and gives 0x4B.  A negative zero keeps its sign bit (0x80), as PyTorch's cast."""
    v = np.array([[1.078125, 0.01263427734375, -0.0, 0.0]], dtype=np.float32)
    codes, s = fp8.quantize_rows(v)
    assert s[0] == np.float32(v[0, 0]) / np.float32(448.0)
    q = v / s[:, None]                                   # NumPy float32 division, IEEE RN
    assert q[0, 1] == 5.25
    ref = torch.from_numpy(q).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(codes, ref)
    assert list(codes[0]) == [0x7E, 0x4A, 0x80, 0x00]
    q_mul = v * (np.float32(1.0) / s)[:, None]
    assert torch.from_numpy(q_mul).to(torch.float8_e4m3fn).view(torch.uint8).numpy()[0, 1] == 0x4B


def _tiny_fp8_layer(T):
    from workloads import TINY, activations, router_weight, expert_weight
    import types
    shape = TINY
    cfg = types.SimpleNamespace(E=shape.E, n_groups=shape.n_groups, topk_groups=shape.topk_groups,
                                topk=shape.topk, routed_scale=shape.routed_scale)
    x = activations(T, shape).float().numpy()
    wr = router_weight(shape).numpy()
    ex = {e: tuple(fp8.Fp8Tensor(expert_weight(shape, e, w).float().numpy()) for w in ("gate", "up", "down"))
          for e in range(shape.E)}
    return shape, cfg, x, wr, ex


def test_fp8_layer_matches_dense_formulation():
    """Gathered per-expert evaluation == every expert on every token weighted by a dense [T, E]
    matrix of the router weights; the layer input is the per-token FP8 quantisation of x."""
    shape, cfg, x, wr, ex = _tiny_fp8_layer(20)
    res = fp8.moe_forward_fp8(x, wr, cfg, lambda e: ex[e])
    r = res["route"]
    xq, xs = fp8.quantize_rows(x)
    np.testing.assert_array_equal(res["xq_codes"], xq)
    xhat = fp8.dequantize_rows(xq, xs)
    dense_w = np.zeros((x.shape[0], shape.E))
    np.put_along_axis(dense_w, r.idx, r.w, axis=1)
    y_all = np.stack([fp8.expert_mlp_fp8(xhat, *ex[e])["y"] for e in range(shape.E)], axis=1)
    np.testing.assert_allclose(res["out"], np.einsum("te,teh->th", dense_w, y_all), rtol=1e-12, atol=1e-12)
    part = fp8.moe_forward_fp8(x, wr, cfg, lambda e: ex[e], tokens=[7, 2, 19])
    np.testing.assert_allclose(part["out"], res["out"][[7, 2, 19]], rtol=1e-12, atol=1e-15)
