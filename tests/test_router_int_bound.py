"""The integer router's documented error bound, checked on the CPU against exact arithmetic.

For T > 64 the library computes each logit from the token row x (BF16) rounded to 22-bit
fixed point and split into three balanced int8 digits, and the router row W (FP32) rounded to
30-bit fixed point and split into four, summed over the 9 digit pairs (i, j) with i + j <= 3
(nvfp4moe.h, route section).  This test rebuilds that computation with Python integers
(exact), checks the digit decompositions, and checks that the result lies within the
documented bound of the exact dot product
    sum|x - x'| |W| + sum|x| |W - W'| + H 2^(e_x + e_W - 28)
    <= 2^(e_x - 23) sum|W| + 2^(e_W - 31) sum|x| + H 2^(e_x + e_W - 28)
(x', W' the fixed-point rows; the FP32 rounding of the final logit is a separate 2^-24 |logit|
term), on random rows and on rows built to stress the scaling: wide exponent spreads,
subnormal BF16 values, zero rows."""
from fractions import Fraction

import numpy as np
import pytest
import torch


def row_exponent(v: np.ndarray) -> int:
    m = float(np.max(np.abs(v)))
    if m == 0.0:
        return -125
    return max(int(np.frexp(m)[1]), -125)


def fixed_point(v: np.ndarray, e: int, bits: int) -> list[int]:
    """RNE(v * 2^(bits - e)) as Python integers (the scaling is exact in float64)."""
    return [int(np.rint(np.ldexp(float(t), bits - e))) for t in v]


def digits(X: int, n: int) -> list[int]:
    """n balanced base-256 digits, most significant first: X = sum_i d_i 2^(8 (n - 1 - i))."""
    out = []
    for _ in range(n - 1):
        d = ((X + 128) & 255) - 128
        out.append(d)
        X = (X - d) >> 8
    out.append(X)
    return out[::-1]


def integer_logit(x: np.ndarray, w: np.ndarray) -> Fraction:
    ex, ew = row_exponent(x), row_exponent(w)
    A = [digits(X, 3) for X in fixed_point(x, ex, 22)]
    B = [digits(W, 4) for W in fixed_point(w, ew, 30)]
    S = 0
    for a, b in zip(A, B):
        for i in range(3):
            for j in range(4):
                if i + j <= 3:
                    S += a[i] * b[j] << (8 * (5 - i - j))
    return Fraction(S) * Fraction(2) ** (ex + ew - 52)


def bound(x: np.ndarray, w: np.ndarray) -> Fraction:
    """The documented bound with the fixed-point roundings of these rows."""
    ex, ew = row_exponent(x), row_exponent(w)
    H = len(x)
    xq = [Fraction(X) * Fraction(2) ** (ex - 22) for X in fixed_point(x, ex, 22)]
    wq = [Fraction(W) * Fraction(2) ** (ew - 30) for W in fixed_point(w, ew, 30)]
    rx = sum(abs(Fraction(float(a)) - q) * abs(Fraction(float(b))) for a, b, q in zip(x, w, xq))
    rw = sum(abs(Fraction(float(a))) * abs(Fraction(float(b)) - q) for a, b, q in zip(x, w, wq))
    return rx + rw + H * Fraction(2) ** (ex + ew - 28)


def bound_worst(x: np.ndarray, w: np.ndarray) -> Fraction:
    """Its worst case over rows with the same exponents and absolute sums."""
    ex, ew = row_exponent(x), row_exponent(w)
    H = len(x)
    sw = sum(Fraction(float(t)).__abs__() for t in w)
    sx = sum(Fraction(float(t)).__abs__() for t in x)
    return Fraction(2) ** (ex - 23) * sw + Fraction(2) ** (ew - 31) * sx + H * Fraction(2) ** (ex + ew - 28)


def exact(x: np.ndarray, w: np.ndarray) -> Fraction:
    return sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(x, w))


def bf16(v) -> np.ndarray:
    return torch.tensor(np.asarray(v, dtype=np.float32)).to(torch.bfloat16).float().numpy().astype(np.float64)


def test_digit_decompositions_are_exact_and_in_range():
    rng = np.random.default_rng(1)
    for n, bits in ((3, 22), (4, 30)):
        for X in list(rng.integers(-(2 ** bits) + 1, 2 ** bits, size=2000)) + [0, 1, -1, 2 ** bits - 1, -(2 ** bits) + 1]:
            X = int(X)
            d = digits(X, n)
            assert sum(t << (8 * (n - 1 - i)) for i, t in enumerate(d)) == X
            assert all(-128 <= t <= 127 for t in d[1:]) and abs(d[0]) <= 64


def test_bf16_rows_are_exact_in_22_bit_fixed_point_within_2_14_of_their_maximum():
    """A BF16 value has 8 significant bits: every element no smaller than 2^-14 of its row's
    largest is represented exactly, so the token-row rounding only touches tiny elements."""
    rng = np.random.default_rng(5)
    x = bf16(rng.standard_normal(4096))
    e = row_exponent(x)
    X = fixed_point(x, e, 22)
    big = np.abs(x) >= 2.0 ** (e - 14)
    assert all(np.ldexp(float(Xi), e - 22) == xi for Xi, xi, b in zip(X, x, big) if b)


def _cases():
    rng = np.random.default_rng(7)
    H = 512
    yield "normal", bf16(rng.standard_normal(H)), rng.standard_normal(H).astype(np.float32) / np.sqrt(H)
    x = bf16(rng.standard_normal(H) * 2.0 ** -20)
    x[17] = 2.0 ** 20
    w = (rng.standard_normal(H) * 2.0 ** -30).astype(np.float32)
    w[3] = 1.0e4
    yield "wide spread", x, w
    yield "subnormal x", bf16(rng.standard_normal(H) * 2.0 ** -130), rng.standard_normal(H).astype(np.float32)
    yield "zero x", np.zeros(H), rng.standard_normal(H).astype(np.float32)
    yield "large H", bf16(rng.standard_normal(5120)), rng.standard_normal(5120).astype(np.float32) / np.sqrt(5120)


@pytest.mark.parametrize("name,x,w", list(_cases()), ids=[c[0] for c in _cases()])
def test_integer_logit_within_documented_bound(name, x, w):
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float32).astype(np.float64)
    err = abs(integer_logit(x, w) - exact(x, w))
    b = bound(x, w)
    assert err <= b, f"{name}: error {float(err):.3g} above bound {float(b):.3g}"
    assert b <= bound_worst(x, w)
    if name == "zero x":
        assert err == 0


def test_bound_is_tighter_than_fp32_accumulation_for_beam_rows():
    """For Beam-like rows (H = 5120, N(0,1) tokens, N(0,1/5120) router) the integer bound is
    below the FP32 accumulation bound 32 * 2^-24 * sum|x W|: by 5x with these rows' roundings,
    and still in its worst case."""
    rng = np.random.default_rng(3)
    H = 5120
    x = bf16(rng.standard_normal(H))
    w = (rng.standard_normal(H) / np.sqrt(H)).astype(np.float32).astype(np.float64)
    fp32_bound = 32 * 2.0 ** -24 * float(np.sum(np.abs(x * w)))
    assert float(bound(x, w)) < fp32_bound / 5
    assert float(bound_worst(x, w)) < fp32_bound
