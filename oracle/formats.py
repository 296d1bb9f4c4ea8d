"""NVFP4 number formats and the quantisation rule, written out plainly.  TEST INFRASTRUCTURE ONLY.

Format ("NVFP4 quantization", section "Quantization scheme"): 4-bit E2M1 codes,
an E4M3 scale for each run of 16 consecutive values along a row, and an FP32
scale for the whole tensor.  A stored value
decodes to ``E2M1[c] * E4M3[S_b] * g``.

The pages do not say how the scales are chosen.  Reading used here (a block
scale is amax/6 relative to a global scale of amax/(6*448)), with every FP32
step one IEEE round-to-nearest-even operation, emulated by one NumPy float32
operation each:

    g    = fp32(A / 2688)           A = max |x| over the tensor; A == 0 -> g = 1
    r_t  = fp32(1 / fp32(6 * g))
    S_b  = E4M3_rne_satfinite(fp32(amax_b * r_t))     (unsigned; may be 0)
    d_b  = fp32(E4M3(S_b) * g);  r_b = 0 if d_b == 0 else fp32(1 / d_b)
    c_i  = E2M1_rne_satfinite(fp32(x_i * r_b))        (sign kept, also on zero)
    byte j of a row = c_{2j} | c_{2j+1} << 4          (even element in the low nibble)

E2M1: 1 sign, 2 exponent bits (bias 1), 1 mantissa bit: magnitudes
{0, 0.5, 1, 1.5, 2, 3, 4, 6}.  E4M3 ("fn" flavour): bias 7, subnormals, no
infinities, 0x7F/0xFF are NaN, largest finite 448.  Both encoders round to the
nearest representable value with ties to the even code and clamp values above
the largest finite magnitude to it.

Scale layouts: "linear" is [rows, cols/16] row-major.  "Swizzled" is the
128x4 tile layout of block-scaled tensor-core operands: rows are padded to a
multiple of 128 and scale columns to a multiple of 4 (padding is zero), tiles
of 128 rows x 4 scale columns are 512 bytes each, ordered row-tile-major then
column tile, and inside a tile the scale of (r, c) sits at byte
``(r % 32) * 16 + (r % 128 // 32) * 4 + c % 4``.
"""
from __future__ import annotations

import numpy as np

F32 = np.float32

# E2M1 magnitudes by code 0..7; codes 8..15 are the negatives (8 is -0).
_E2M1_MAG = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)
E2M1_VALUES = np.concatenate([_E2M1_MAG, -_E2M1_MAG])


def _e4m3_value(code: int) -> float:
    """Value of one E4M3 byte from its bit fields (bias 7, subnormals, NaN at S.1111.111)."""
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * (m / 8.0) * 2.0 ** (-6)
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


_E4M3 = np.array([_e4m3_value(c) for c in range(256)], dtype=np.float64)
E4M3_MAX = 448.0


def e4m3_table() -> np.ndarray:
    """FP64 value of every E4M3 byte 0..255."""
    return _E4M3.copy()


def e2m1_decode(codes: np.ndarray) -> np.ndarray:
    return E2M1_VALUES[np.asarray(codes, dtype=np.int64) & 0xF]


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    return _E4M3[np.asarray(codes, dtype=np.int64) & 0xFF]


def _nearest_even(v: np.ndarray, grid: np.ndarray) -> np.ndarray:
    """Index into the increasing ``grid`` nearest to each v >= 0 (ties to the even index).

    Values above the last grid point clamp to it (saturation).
    """
    v = np.asarray(v, dtype=np.float64)
    hi = np.searchsorted(grid, v, side="left")           # grid[hi-1] < v <= grid[hi]
    hi = np.clip(hi, 0, len(grid) - 1)
    lo = np.clip(hi - 1, 0, len(grid) - 1)
    d_lo = v - grid[lo]
    d_hi = grid[hi] - v
    pick = np.where(d_lo < d_hi, lo, hi)
    tie = d_lo == d_hi
    pick = np.where(tie, np.where(lo % 2 == 0, lo, hi), pick)
    pick = np.where(v >= grid[-1], len(grid) - 1, pick)
    return pick


_E4M3_POS = _E4M3[:0x7F]            # codes 0x00..0x7E, increasing, 0 .. 448


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    """Unsigned E4M3 byte nearest to each v >= 0 (ties to even, clamped to 448); NaN -> 0x7F."""
    v = np.asarray(v, dtype=np.float64)
    if np.any(v < 0):
        raise ValueError("block scales are unsigned")
    code = _nearest_even(np.nan_to_num(v, nan=0.0), _E4M3_POS).astype(np.uint8)
    return np.where(np.isnan(v), np.uint8(0x7F), code).astype(np.uint8)


def e2m1_encode(v: np.ndarray) -> np.ndarray:
    """E2M1 code (0..15) nearest to each finite v (ties to even, clamped to +-6, sign kept).

    The nearest-value search over the 8 magnitudes is written as a count of the
    midpoints between consecutive grid values that |v| passes: between codes i
    and i+1 the midpoint is passed when |v| > mid for even i (a tie stays on the
    even code i) and when |v| >= mid for odd i (a tie moves to the even code i+1).
    """
    v = np.asarray(v)
    if not np.all(np.isfinite(v)):
        raise ValueError("E2M1 encoding needs finite inputs")
    mag = np.abs(v)
    code = np.zeros(v.shape, dtype=np.uint8)
    for i in range(7):
        mid = (_E2M1_MAG[i] + _E2M1_MAG[i + 1]) / 2
        code += (mag > mid) if i % 2 == 0 else (mag >= mid)
    code[np.signbit(v)] |= np.uint8(8)
    return code


def global_scale(amax) -> np.float32:
    """g = fp32(A / 2688), or 1 when A == 0.  A must be finite."""
    a = F32(amax)
    if not np.isfinite(a):
        raise ValueError("non-finite tensor amax")
    if a == 0:
        return F32(1.0)
    return F32(a / F32(2688.0))


def quantize(x, g=None):
    """Quantise a [rows, cols] float32 tensor (cols % 16 == 0) by the rule in the module docstring.

    Returns (codes uint8 [rows, cols/2], scales uint8 [rows, cols/16] linear, g float32).
    ``g`` given: used as is (a static scale); None: computed from the tensor's amax.
    """
    x = np.asarray(x)
    if x.dtype != np.float32:
        raise TypeError("quantize expects float32 values (BF16 inputs widen exactly)")
    rows, cols = x.shape
    if cols % 16:
        raise ValueError("cols must be a multiple of 16")
    if g is None:
        g = global_scale(np.max(np.abs(x)) if x.size else 0.0)
    g = F32(g)
    r_t = F32(1.0) / (F32(6.0) * g)
    xb = x.reshape(rows, cols // 16, 16)
    amax_b = np.max(np.abs(xb), axis=2) if x.size else np.zeros((rows, cols // 16), F32)
    S = e4m3_encode((amax_b * r_t).astype(F32))
    d = (e4m3_decode(S).astype(F32) * g).astype(F32)
    with np.errstate(divide="ignore"):
        r_b = np.where(d == 0, F32(0.0), F32(1.0) / d).astype(F32)
    v = (xb * r_b[:, :, None]).astype(F32)
    c = e2m1_encode(v).reshape(rows, cols)
    codes = (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)
    return codes, S.reshape(rows, cols // 16), g


def unpack_codes(codes: np.ndarray) -> np.ndarray:
    """[rows, cols/2] packed bytes -> [rows, cols] codes (low nibble first)."""
    codes = np.asarray(codes, dtype=np.uint8)
    out = np.empty((codes.shape[0], codes.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = codes & 0xF
    out[:, 1::2] = codes >> 4
    return out


def dequantize(codes, scales, g) -> np.ndarray:
    """FP64 [rows, cols] values E2M1[c] * E4M3[S] * g (exact in FP64)."""
    c = unpack_codes(codes)
    rows, cols = c.shape
    s = e4m3_decode(np.asarray(scales)).reshape(rows, cols // 16)
    return e2m1_decode(c) * np.repeat(s, 16, axis=1) * np.float64(F32(g))


def swizzled_scale_bytes(rows: int, cols16: int) -> int:
    """Size of the swizzled scale array for ``rows`` rows and ``cols16`` scale columns."""
    return (-(-rows // 128) * 128) * (-(-cols16 // 4) * 4)


def swizzle_scales(linear: np.ndarray) -> np.ndarray:
    """Linear [rows, cols16] scales -> flat swizzled uint8 array (zero padding)."""
    linear = np.asarray(linear, dtype=np.uint8)
    rows, cols16 = linear.shape
    n_ct = -(-cols16 // 4)
    out = np.zeros(swizzled_scale_bytes(rows, cols16), dtype=np.uint8)
    r = np.arange(rows)[:, None]
    c = np.arange(cols16)[None, :]
    off = (r // 128) * (n_ct * 512) + (c // 4) * 512 + (r % 32) * 16 + (r % 128 // 32) * 4 + c % 4
    out[off] = linear
    return out


def unswizzle_scales(flat: np.ndarray, rows: int, cols16: int) -> np.ndarray:
    flat = np.asarray(flat, dtype=np.uint8)
    n_ct = -(-cols16 // 4)
    r = np.arange(rows)[:, None]
    c = np.arange(cols16)[None, :]
    off = (r // 128) * (n_ct * 512) + (c // 4) * 512 + (r % 32) * 16 + (r % 128 // 32) * 4 + c % 4
    return flat[off]


def nvfp4_tensor_bytes(rows: int, cols: int) -> int:
    """Bytes of an NVFP4 tensor: 4-bit codes plus one 8-bit scale per 16 values (no global)."""
    return rows * cols // 2 + rows * cols // 16
