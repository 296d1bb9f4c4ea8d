"""Pins of oracle/local_hessian.py (the block-scale search of "NVFP4 quantization", section
"Quantization method"): with no candidates besides the round-to-nearest scale it is the
quantisation rule itself; it never does worse than that scale; a hand-built block whose exact
answer is a non-default scale; invariance to the scale of H; zero blocks."""
import numpy as np

import oracle


def _spd(nb, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((64, nb * 16)) * (1 + rng.random(nb * 16))
    return oracle.hessian_blocks(x)


def _weights(rows, cols, seed):
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((rows, cols)).astype(np.float32) * np.float32(0.02)
    return oracle.moe._bf16_round(w.astype(np.float64)).astype(np.float32)


def test_no_candidates_is_the_rounding_rule():
    w = _weights(8, 64, 0)
    codes, S, g, errs, cands = oracle.quantize_local_hessian(w, _spd(4, 1), m=0)
    c_ref, s_ref, g_ref = oracle.quantize(w)
    np.testing.assert_array_equal(codes, c_ref)
    np.testing.assert_array_equal(S, s_ref)
    assert g == g_ref


def test_search_never_worse_than_rounding_rule():
    w = _weights(16, 128, 2)
    H = _spd(8, 3)
    codes, S, g, errs, cands = oracle.quantize_local_hessian(w, H, m=4)
    chosen = errs.min(axis=2)
    assert np.all(chosen <= errs[..., 0])
    # the chosen scale is the first minimum in the visiting order
    k = np.argmin(errs, axis=2)
    np.testing.assert_array_equal(S, np.take_along_axis(cands, k[..., None], axis=2)[..., 0])
    # and it usually helps: strictly better on some blocks
    assert np.any(chosen < errs[..., 0])


def test_worked_block_takes_the_exact_scale():
    """Tensor amax 168 -> g = 168/2688 = 1/16, r_t = 8/3.  Block [2.75, 0, ...]: the rounding
    rule gives S0 = E4M3(2.75 * 8/3 = 7.33) = 7.5 (code 79), d = 0.46875, 2.75 / d = 5.87 ->
    E2M1 6 -> 2.8125 (error 0.0625).  Scale 11 (code 83 = S0 + 4): d = 0.6875, 2.75 / d = 4
    exactly -> error 0.  With H weighting only that element the search must take code 83."""
    w = np.zeros((2, 16), dtype=np.float32)
    w[0, 0] = 168.0
    w[1, 0] = 2.75
    H = np.zeros((1, 16, 16))
    H[0, 0, 0] = 1.0
    codes, S, g, errs, cands = oracle.quantize_local_hessian(w, H, m=4)
    assert g == np.float32(1 / 16)
    assert cands[1, 0, 0] == 79 and oracle.e4m3_decode(np.uint8(79)) == 7.5
    assert S[1, 0] == 83 and oracle.e4m3_decode(np.uint8(83)) == 11.0
    assert errs[1, 0, 0] == 0.0625 ** 2
    deq = oracle.dequantize(codes, S, g)
    assert deq[1, 0] == 2.75


def test_invariant_to_the_scale_of_h():
    w = _weights(8, 64, 4)
    H = _spd(4, 5)
    a = oracle.quantize_local_hessian(w, H, m=3)
    b = oracle.quantize_local_hessian(w, H * 37.0, m=3)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_zero_blocks_stay_zero():
    w = _weights(4, 64, 6)
    w[:, 16:32] = 0.0
    codes, S, g, errs, cands = oracle.quantize_local_hessian(w, _spd(4, 7), m=4)
    assert np.all(S[:, 1] == 0)
    assert np.all(oracle.formats.unpack_codes(codes)[:, 16:32] == 0)


def test_candidate_order():
    assert oracle.candidate_offsets(2) == [0, -1, 1, -2, 2]


def test_zero_hessian_keeps_the_rounding_rule():
    """With H_b = 0 every candidate's error is 0; a candidate replaces the best only when strictly
    better, so the search keeps the round-to-nearest scale S0 (the first visited)."""
    w = _weights(8, 64, 8)
    codes, S, g, errs, cands = oracle.quantize_local_hessian(w, np.zeros((4, 16, 16)), m=4)
    assert np.all(errs == 0)
    c_ref, s_ref, _ = oracle.quantize(w)
    np.testing.assert_array_equal(S, s_ref)
    np.testing.assert_array_equal(codes, c_ref)


def test_h_weighting_decides():
    """The block [2.75, 1.875, 0.1875, 0, ...] under tensor amax 168 (g = 1/16): S0 = code 79
    (7.5, d = 0.46875) represents 1.875 = 4 d exactly and misses 2.75 by 0.0625; code 83 (11,
    d = 0.6875) represents 2.75 = 4 d exactly and misses 1.875 by 0.1875 (1.875 / d = 2.73 ->
    E2M1 3); of the codes 75 .. 83 only 76 (6, d = 0.375, below S0) represents 0.1875 = d / 2
    exactly.  Weighting only element 0 the search must take 83, only element 2 it must take
    76, and only element 1 it must keep 79 (code 82, d = 0.625, also represents 1.875 exactly,
    as 3 d: that tie keeps S0, the first visited)."""
    w = np.zeros((2, 16), dtype=np.float32)
    w[0, 0] = 168.0
    w[1, 0], w[1, 1], w[1, 2] = 2.75, 1.875, 0.1875
    for k, want in ((0, 83), (1, 79), (2, 76)):
        H = np.zeros((1, 16, 16))
        H[0, k, k] = 1.0
        codes, S, g, errs, cands = oracle.quantize_local_hessian(w, H, m=4)
        assert g == np.float32(1 / 16) and cands[1, 0, 0] == 79
        assert S[1, 0] == want, (k, S[1, 0])
        deq = oracle.dequantize(codes, S, g)
        assert deq[1, k] == w[1, k]


def test_hessian_blocks_by_loops():
    """H_b[i, j] = sum over tokens of x[n, 16 b + i] x[n, 16 b + j], by plain loops."""
    rng = np.random.default_rng(9)
    x = rng.standard_normal((5, 48))
    H = oracle.hessian_blocks(x)
    assert H.shape == (3, 16, 16)
    for b in range(3):
        for i in range(16):
            for j in range(16):
                want = sum(x[n, 16 * b + i] * x[n, 16 * b + j] for n in range(5))
                assert abs(H[b, i, j] - want) <= 1e-12 * max(1.0, abs(want))
