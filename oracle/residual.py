"""The MoE block's neighbours on the residual stream: the RMSNorm that produces the layer
input and the weighted residual add of the layer output.  TEST INFRASTRUCTURE ONLY.

Follows "Reflection releases Beam ...", section "Residual stream and numerical decisions":
the input embedding is step 1 of the residual stream; at step k a sublayer output is added
with weight 1/sqrt(k) while the existing stream is kept with weight sqrt((k-1)/k), so the
squares of the two weights sum to one and, after n steps, the embedding and every sublayer
output carry the same weight 1/sqrt(n); norms are computed in FP32.

Readings where the pages are silent:

* The norm before the MoE block is an RMSNorm with a per-channel weight gamma:
  x = h / sqrt(mean(h^2) + eps) * gamma, eps given by the caller.
* Its arithmetic: the mean of squares and the reciprocal root r in FP64 (from BF16 h every
  square is exact), r rounded to FP32 once, then two FP32 multiplies per element,
  x = fp32(fp32(h * r) * gamma), rounded to BF16 (round-to-nearest-even): the layer input
  is a BF16 tensor like the residual stream.
* The weights a = sqrt((k-1)/k) and b = 1/sqrt(k) are FP64 values rounded to FP32, and the
  new stream is h' = a*h + b*moe(x), rounded to BF16 once.
"""
from __future__ import annotations

import numpy as np

from .moe import _bf16_round


def rmsnorm_scale(h, eps: float) -> np.ndarray:
    """r[t] = 1 / sqrt(mean_j h[t, j]^2 + eps) in FP64, returned rounded to FP32."""
    h = np.asarray(h, dtype=np.float64)
    ms = np.mean(h * h, axis=1)
    return (1.0 / np.sqrt(ms + float(eps))).astype(np.float32)


def rmsnorm(h, gamma, eps: float) -> np.ndarray:
    """The layer input x = bf16(fp32(fp32(h * r) * gamma)) as float32 values [T, H].

    h: [T, H] values of a BF16 tensor; gamma: [H] FP32."""
    h32 = np.asarray(h, dtype=np.float32)
    r = rmsnorm_scale(h32, eps)
    y = (h32 * r[:, None]).astype(np.float32)              # one FP32 multiply, RN
    y = (y * np.asarray(gamma, dtype=np.float32)[None, :]).astype(np.float32)
    return _bf16_round(y.astype(np.float64)).astype(np.float32)


def residual_weights(k: int) -> tuple[np.float32, np.float32]:
    """(a, b) = (sqrt((k-1)/k), 1/sqrt(k)) as FP32, for residual step k >= 1."""
    if k < 1:
        raise ValueError("residual step k starts at 1")
    return np.float32(np.sqrt((k - 1) / k)), np.float32(1.0 / np.sqrt(k))


def residual_add(h, moe_out, k: int) -> np.ndarray:
    """h' = a*h + b*moe_out in FP64 (a, b the FP32 weights of step k), not rounded."""
    a, b = residual_weights(k)
    return float(a) * np.asarray(h, dtype=np.float64) + float(b) * np.asarray(moe_out, dtype=np.float64)
