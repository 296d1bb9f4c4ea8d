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
