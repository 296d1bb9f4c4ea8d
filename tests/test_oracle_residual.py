"""Pins of oracle/residual.py (RMSNorm before the MoE block, weighted residual add after it)
against the page's statement ("Reflection releases Beam ...", section "Residual stream and
numerical decisions"), closed forms and one value worked by hand."""
import math

import numpy as np
import pytest

import oracle


def test_step_one_keeps_only_the_sublayer_and_step_two_halves():
    assert oracle.residual_weights(1) == (np.float32(0.0), np.float32(1.0))
    a, b = oracle.residual_weights(2)
    assert a == b == np.float32(math.sqrt(0.5))
    with pytest.raises(ValueError):
        oracle.residual_weights(0)


@pytest.mark.parametrize("k", [2, 3, 7, 52])
def test_weights_squares_sum_to_one(k):
    a, b = oracle.residual_weights(k)
    assert abs(float(a) ** 2 + float(b) ** 2 - 1.0) < 4e-7


@pytest.mark.parametrize("n", [2, 5, 49, 52])
def test_equal_contributions_after_n_steps(n):
    """The page: after all additions the input embedding and every sublayer output contribute
    equally to the final hidden state.  Composing the weights of steps 2..n must give each of
    them 1/sqrt(n) (to FP32 rounding of the per-step weights)."""
    contrib = [1.0]                         # the embedding, step 1
    for k in range(2, n + 1):
        a, b = (float(v) for v in oracle.residual_weights(k))
        contrib = [c * a for c in contrib] + [b]
    expect = 1.0 / math.sqrt(n)
    assert np.allclose(contrib, expect, rtol=2e-6 * n, atol=0)


def test_residual_add_is_the_weighted_sum():
    rng = np.random.default_rng(0)
    h, y = rng.standard_normal((3, 16)), rng.standard_normal((3, 16))
    np.testing.assert_array_equal(oracle.residual_add(h, y, 1), y)
    a, b = oracle.residual_weights(5)
    np.testing.assert_allclose(oracle.residual_add(h, y, 5), float(a) * h + float(b) * y, rtol=0, atol=0)


def test_rmsnorm_worked_value():
    """h = [3, 4, 0, 0], gamma = 1, eps = 0: mean(h^2) = 25/4, r = fp32(0.4);
    3 * r = 1.2000000178..., FP32 1.2000000477; BF16 (step 2^-7 near 1.2): 154/128 = 1.203125;
    4 * r -> 1.6000000238 -> 205/128 = 1.6015625."""
    x = oracle.rmsnorm(np.array([[3.0, 4.0, 0.0, 0.0]]), np.ones(4), 0.0)
    np.testing.assert_array_equal(x, np.array([[1.203125, 1.6015625, 0.0, 0.0]], dtype=np.float32))


def test_rmsnorm_constant_rows_give_sign_times_gamma():
    gamma = np.array([1.0, -2.0, 0.375, 96.0], dtype=np.float32)        # BF16-exact values
    h = np.array([[4.0] * 4, [-0.25] * 4, [2.0 ** -10] * 4], dtype=np.float32)
    x = oracle.rmsnorm(h, gamma, 0.0)
    np.testing.assert_array_equal(x, np.sign(h) * gamma[None, :])


def test_rmsnorm_scale_invariance_and_zero_rows():
    rng = np.random.default_rng(1)
    h = oracle.moe._bf16_round(rng.standard_normal((4, 64))).astype(np.float32)
    gamma = oracle.moe._bf16_round(1 + 0.1 * rng.standard_normal(64)).astype(np.float32)
    x = oracle.rmsnorm(h, gamma, 0.0)
    for s in (-6, 3, 20):
        np.testing.assert_array_equal(oracle.rmsnorm(h * np.float32(2.0 ** s), gamma, 0.0), x)
    z = oracle.rmsnorm(np.zeros((2, 64), dtype=np.float32), gamma, 1e-6)
    np.testing.assert_array_equal(z, np.zeros((2, 64), dtype=np.float32))
    # eps only lowers the scale
    assert np.all(oracle.rmsnorm_scale(h, 1e-2) <= oracle.rmsnorm_scale(h, 0.0))


def test_rmsnorm_eps_inside_the_root():
    """A constant row of ones with eps = 3: mean(h^2) + eps = 4, r = 1/2 exactly, so
    x = gamma / 2 (BF16-exact gammas)."""
    gamma = np.array([1.0, -2.0, 0.375, 96.0], dtype=np.float32)
    x = oracle.rmsnorm(np.ones((1, 4), dtype=np.float32), gamma, 3.0)
    np.testing.assert_array_equal(x[0], gamma / 2)
    assert oracle.rmsnorm_scale(np.ones((1, 4)), 3.0)[0] == np.float32(0.5)
