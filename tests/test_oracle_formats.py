"""Pins for the oracle's NVFP4 formats and quantisation rule (CPU only).

Each check ties the oracle to something other than itself: a bit-field
derivation of E2M1, torch's float8_e4m3fn casts (a library routine),
brute-force nearest-value searches, hand-worked layout offsets, closed-form
invariants of the rule, and the size figures the pages print.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import formats as F
from tests.conftest import read_golden


# ---------------------------------------------------------------- E2M1 ----

def _e2m1_from_bits(code):
    """E2M1 by its bit fields: sign, 2 exponent bits with bias 1, 1 mantissa bit."""
    s = -1.0 if code & 8 else 1.0
    e = (code >> 1) & 3
    m = code & 1
    if e == 0:
        return s * (m / 2.0)              # subnormal: 0.m * 2^(1-1)
    return s * (1.0 + m / 2.0) * 2.0 ** (e - 1)


def test_e2m1_table_matches_bit_definition_and_golden():
    gold = {int(c): float(v) for c, v in read_golden("e2m1_grid.txt")}
    for code in range(16):
        v = oracle.e2m1_decode(np.array([code]))[0]
        assert v == _e2m1_from_bits(code) == gold[code]
        assert math.copysign(1, v) == math.copysign(1, gold[code])


def test_e2m1_ties_golden():
    for inp, code in read_golden("e2m1_ties.txt"):
        got = oracle.e2m1_encode(np.array([np.float32(inp)]))[0]
        assert int(got) == int(code), inp


def _e2m1_brute(v):
    """Nearest E2M1 magnitude by exhaustive search, ties to the even code, clamp to 6."""
    mag = abs(v)
    best = None
    for code in range(8):
        d = abs(mag - _e2m1_from_bits(code))
        if best is None or d < best[0] or (d == best[0] and code % 2 == 0):
            best = (d, code)
    code = best[1] if mag <= 6.0 else 7
    return code | (8 if math.copysign(1, v) < 0 else 0)


def test_e2m1_encode_matches_brute_force_dense_sweep():
    grid = sorted({abs(_e2m1_from_bits(c)) for c in range(8)})
    pts = [0.0, 6.0, 6.5, 100.0]
    for a, b in zip(grid[:-1], grid[1:]):
        mid = np.float32((a + b) / 2)
        pts += [mid, np.nextafter(mid, np.float32(0)), np.nextafter(mid, np.float32(10))]
    rng = np.random.default_rng(1)
    pts += list(rng.uniform(0, 7, 2000))
    v = np.array(pts, dtype=np.float32)
    v = np.concatenate([v, -v])
    got = oracle.e2m1_encode(v)
    want = np.array([_e2m1_brute(float(x)) for x in v])
    np.testing.assert_array_equal(got, want)


# ---------------------------------------------------------------- E4M3 ----

def test_e4m3_table_matches_torch_float8():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    tab = oracle.e4m3_table()
    np.testing.assert_array_equal(np.isnan(tab), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(tab[ok], ref[ok])


def test_e4m3_points_golden():
    g = {k: float(v) for k, v in read_golden("e4m3_points.txt")}
    tab = oracle.e4m3_table()
    pos = tab[:128]
    assert np.nanmax(tab) == g["max_finite"] == F.E4M3_MAX
    assert tab[int(g["max_finite_code"])] == g["max_finite"]
    assert np.isnan(tab[int(g["nan_code"])]) and np.isnan(tab[int(g["nan_code"]) | 0x80])
    assert tab[1] == g["min_subnormal"] and tab[8] == g["min_normal"]
    assert np.sum(np.isfinite(pos)) == g["finite_nonneg_codes"]


def test_e4m3_encode_matches_torch_rne_below_saturation():
    grid = oracle.e4m3_table()[:127]
    mids = (grid[:-1] + grid[1:]) / 2
    pts = [grid, mids, np.nextafter(mids.astype(np.float32), np.float32(0)),
           np.nextafter(mids.astype(np.float32), np.float32(1000)),
           np.random.default_rng(2).uniform(0, 460, 20000),
           np.exp(np.random.default_rng(3).uniform(-12, 6, 20000))]
    v = np.concatenate([np.asarray(p, dtype=np.float32) for p in pts])
    v = v[v < 464.0]                   # torch's cast has no saturation above the 448/480 midpoint
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(oracle.e4m3_encode(v), ref)


def test_e4m3_encode_saturates():
    v = np.array([448.0, 463.9, 464.0, 480.0, 1e6, 3e38], dtype=np.float32)
    assert list(oracle.e4m3_encode(v)) == [126] * 6
    assert oracle.e4m3_encode(np.array([np.nan]))[0] == 0x7F


# ------------------------------------------------------- quantise rule ----

def _blocks(n_rows=64, cols=256, seed=0, scale=1.0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n_rows, cols)) * scale
    # a spread of block magnitudes, an all-zero block and a negative-zero block
    x *= np.repeat(np.exp(rng.uniform(-4, 2, (n_rows, cols // 16))), 16, axis=1)
    x[3, 16:32] = 0.0
    x[4, 32:48] = -0.0
    return torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()


def test_global_scale_definition():
    for a in [1.0, 3.5, 2688.0, 1e-3, 7.25e5]:
        g = oracle.global_scale(a)
        assert g == np.float32(np.float32(a) / np.float32(2688.0))
        assert abs(float(g) * 6 * 448 - a) <= a * 2.0 ** -23
    assert oracle.global_scale(0.0) == 1.0
    with pytest.raises(ValueError):
        oracle.global_scale(np.inf)


def test_quantize_block_scale_is_nearest_e4m3_by_brute_force():
    x = _blocks()
    codes, S, g = oracle.quantize(x)
    q = (np.abs(x.reshape(64, 16, 16)).max(axis=2) * (np.float32(1) / (np.float32(6) * g))).astype(np.float32)
    tab = oracle.e4m3_table()[:127]
    for (i, j), qq in np.ndenumerate(q):
        d = np.abs(tab - float(qq))
        cands = np.flatnonzero(d == d.min())
        want = cands[0] if len(cands) == 1 else [c for c in cands if c % 2 == 0][0]
        assert S[i, j] == min(want, 126)


def test_quantize_max_block_hits_448_and_decodes_to_amax():
    x = _blocks()
    codes, S, g = oracle.quantize(x)
    A = np.abs(x).max()
    r, c = np.unravel_index(np.argmax(np.abs(x)), x.shape)
    assert S[r, c // 16] == 126                               # E4M3 448
    xh = oracle.dequantize(codes, S, g)
    assert abs(abs(xh[r, c]) - A) <= A * 2.0 ** -22           # 6 * 448 * g == A up to g's rounding
    assert abs(xh[r, c]) == 6 * 448 * float(g)


def test_quantize_error_bound_and_zero_blocks():
    x = _blocks()
    codes, S, g = oracle.quantize(x)
    xh = oracle.dequantize(codes, S, g)
    d = np.repeat(oracle.e4m3_decode(S) * float(g), 16, axis=1)
    mag = np.abs(xh) / np.where(d == 0, 1, d)
    half_step = np.where(mag < 2, 0.25, np.where(mag < 4, 0.5, 1.0))
    unsat = np.abs(x) <= 6 * d
    err = np.abs(xh - x)
    assert np.all(err[unsat] <= half_step[unsat] * d[unsat] * (1 + 2 ** -20) + 1e-30)
    assert S[3, 1] == 0 and np.all(codes[3, 8:16] == 0)
    assert S[4, 2] == 0 and np.all(codes[4, 16:24] == 0x88)     # -0 keeps its sign bit


def test_quantize_sign_symmetry():
    x = _blocks(seed=5)
    c1, s1, g1 = oracle.quantize(x)
    c2, s2, g2 = oracle.quantize(-x)
    assert g1 == g2
    np.testing.assert_array_equal(s1, s2)
    np.testing.assert_array_equal(c2, c1 ^ 0x88)


def test_quantize_idempotent_on_normal_scales():
    x = _blocks(seed=7)
    codes, S, g = oracle.quantize(x)
    xh = oracle.dequantize(codes, S, g).astype(np.float32)
    c2, s2, _ = oracle.quantize(xh, g=g)
    normal = np.repeat(oracle.e4m3_decode(S) >= 2.0 ** -6, 8, axis=1)
    np.testing.assert_array_equal(s2[S >= 8], S[S >= 8])
    np.testing.assert_array_equal(c2[normal], codes[normal])


def test_quantize_static_scale_saturates():
    x = np.full((1, 16), 10.0, dtype=np.float32)
    codes, S, g = oracle.quantize(x, g=np.float32(1e-3))      # calibrated range far below 10
    assert S[0, 0] == 126 and np.all(codes == 0x77)


def test_pack_order_low_nibble_is_even_element():
    x = np.zeros((1, 16), dtype=np.float32)
    x[0, 0] = 6.0          # code 7 in the low nibble of byte 0
    x[0, 1] = -3.0         # code 13 in the high nibble of byte 0
    codes, S, g = oracle.quantize(x)
    assert codes[0, 0] == (7 | (13 << 4))


# -------------------------------------------------------------- layout ----

def test_swizzle_offsets_golden():
    lin = np.zeros((256, 8), dtype=np.uint8)
    rows = read_golden("swizzle_offsets.txt")
    for k, (r, c, _) in enumerate(rows):
        lin[int(r), int(c)] = k + 1
    flat = oracle.swizzle_scales(lin)
    assert flat.size == 2048
    for k, (r, c, off) in enumerate(rows):
        assert flat[int(off)] == k + 1


def test_swizzle_roundtrip_and_padding():
    rng = np.random.default_rng(0)
    lin = rng.integers(1, 255, (200, 12), dtype=np.uint8)
    flat = oracle.swizzle_scales(lin)
    assert flat.size == 256 * 12
    np.testing.assert_array_equal(oracle.unswizzle_scales(flat, 200, 12), lin)
    assert np.count_nonzero(flat) == lin.size                  # padding rows are zero


# --------------------------------------------------------------- sizes ----

def test_sizes_match_pages():
    g = {r[0]: float(r[1]) for r in read_golden("model_sizes.txt")}
    H, I, E = 5120, 2560, 256
    params = 3 * H * I
    assert params == 39_321_600 and abs(params - g["expert_params_approx"]) / params < 0.01
    expert_bytes = oracle.nvfp4_tensor_bytes(2 * I, H) + oracle.nvfp4_tensor_bytes(H, I)
    assert expert_bytes / params == g["bytes_per_param"] == 0.5625
    assert expert_bytes == 22_118_400 and abs(expert_bytes - g["expert_bytes_approx"]) / 22e6 < 0.01
    layer = E * expert_bytes + g["attention_bytes_approx"]
    assert abs(layer - g["moe_layer_file_bytes"]) / g["moe_layer_file_bytes"] < 0.01
    # whole checkpoint: expert params in NVFP4, the rest BF16 (the BF16 size fixes the total)
    total = g["bf16_checkpoint_gib"] * 2 ** 30 / 2
    expert_params = g["moe_layers"] * g["experts_per_layer"] * params
    rest = total - expert_params
    nvfp4 = expert_params * 0.5625 + rest * 2
    assert abs(nvfp4 / 2 ** 30 - g["nvfp4_checkpoint_gib"]) < 1.0
    assert abs(nvfp4 / 1e9 - g["nvfp4_checkpoint_gb"]) < 0.5
    assert abs(expert_params / total - g["expert_param_share"]) < 0.001
    assert abs(total - g["total_params_approx"]) / total < 0.002
    active = g["moe_layers"] * g["active_experts"] * params + rest
    assert abs(active - g["active_params_approx"]) / active < 0.05
