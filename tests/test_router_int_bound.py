"""The integer router's documented error bound, checked on the CPU against exact arithmetic.

For T > 64 the library computes each logit from the token row x (BF16) and the router row W
(FP32) rounded to 30-bit fixed point, split into four balanced int8 digits, and summed over
the 13 digit pairs (i, j) with i + j <= 4 (nvfp4moe.h, route section).  This test rebuilds
that computation with Python integers (exact), checks the digit decomposition, and checks
that the result lies within the documented bound of the exact dot product
    2^(e_x - 31) sum|W| + 2^(e_W - 31) sum|x| + H 2^(e_x + e_W - 36)
(the FP32 rounding of the final logit is a separate 2^-24 |logit| term), on random rows and on
rows built to stress the scaling: wide exponent spreads, subnormal BF16 values, zero rows."""
from fractions import Fraction

import numpy as np
import pytest
import torch


def row_exponent(v: np.ndarray) -> int:
    m = float(np.max(np.abs(v)))
    if m == 0.0:
        return -125
    return max(int(np.frexp(m)[1]), -125)


def fixed_point(v: np.ndarray, e: int) -> list[int]:
    """RNE(v * 2^(30 - e)) as Python integers (the scaling is exact in float64)."""
    return [int(np.rint(np.ldexp(float(t), 30 - e))) for t in v]


def digits(X: int) -> list[int]:
    """Balanced base-256 digits, most significant first: X = d0 2^24 + d1 2^16 + d2 2^8 + d3."""
    out = []
    for _ in range(3):
        d = ((X + 128) & 255) - 128
        out.append(d)
        X = (X - d) >> 8
    out.append(X)
    return out[::-1]


def integer_logit(x: np.ndarray, w: np.ndarray) -> Fraction:
    ex, ew = row_exponent(x), row_exponent(w)
    A = [digits(X) for X in fixed_point(x, ex)]
    B = [digits(W) for W in fixed_point(w, ew)]
    S = 0
    for a, b in zip(A, B):
        for i in range(4):
            for j in range(4):
                if i + j <= 4:
                    S += a[i] * b[j] << (8 * (6 - i - j))
    return Fraction(S) * Fraction(2) ** (ex + ew - 60)


def bound(x: np.ndarray, w: np.ndarray) -> Fraction:
    ex, ew = row_exponent(x), row_exponent(w)
    H = len(x)
    sw = sum(Fraction(float(t)).__abs__() for t in w)
    sx = sum(Fraction(float(t)).__abs__() for t in x)
    return Fraction(2) ** (ex - 31) * sw + Fraction(2) ** (ew - 31) * sx + H * Fraction(2) ** (ex + ew - 36)


def exact(x: np.ndarray, w: np.ndarray) -> Fraction:
    return sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(x, w))


def bf16(v) -> np.ndarray:
    return torch.tensor(np.asarray(v, dtype=np.float32)).to(torch.bfloat16).float().numpy().astype(np.float64)


def test_digit_decomposition_is_exact_and_in_range():
    rng = np.random.default_rng(1)
    for X in list(rng.integers(-(2 ** 30) + 1, 2 ** 30, size=2000)) + [0, 1, -1, 2 ** 30 - 1, -(2 ** 30) + 1]:
        X = int(X)
        d = digits(X)
        assert (d[0] << 24) + (d[1] << 16) + (d[2] << 8) + d[3] == X
        assert all(-128 <= t <= 127 for t in d[1:]) and abs(d[0]) <= 64


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
    if name == "zero x":
        assert err == 0


def test_bound_is_much_tighter_than_fp32_accumulation_for_beam_rows():
    """For Beam-like rows (H = 5120, N(0,1) tokens, N(0,1/5120) router) the integer bound is
    far below the FP32 accumulation bound 32 * 2^-24 * sum|x W|."""
    rng = np.random.default_rng(3)
    H = 5120
    x = bf16(rng.standard_normal(H))
    w = (rng.standard_normal(H) / np.sqrt(H)).astype(np.float32).astype(np.float64)
    fp32_bound = 32 * 2.0 ** -24 * float(np.sum(np.abs(x * w)))
    assert float(bound(x, w)) < fp32_bound / 50
