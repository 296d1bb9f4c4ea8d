"""The FP8 W8A8 variant of the routed-expert layer.  TEST INFRASTRUCTURE ONLY.

Follows "FP8 quantization", section "Quantization scheme": FP8 E4M3 weights and input
activations; each weight output channel has a fixed scale; activation scales are computed
per token at run time; the expert gate, up and down projections are quantised (the router
is not).  Section "Quantization method": round-to-nearest, weights divided by their scales
and rounded to the nearest FP8 value.

Readings where the pages are silent:

* The scale of a row (a weight output channel, or a token's activation row) is
  s = fp32(amax / 448), 448 being the largest E4M3 value; a row whose amax is 0 takes s = 1.
* code = E4M3_rne_satfinite(fp32(v / s)) with an IEEE division; signed (E4M3 sign bit).
* The input of the down projection is the SwiGLU product h, rounded to FP32, quantised per
  (token, slot) row with its own scale, like the layer input.
* Everything else (routing, grouping, the weighted combine, BF16 output) is the NVFP4
  layer's; the MLP is evaluated in FP64 on dequantised operands.
"""
from __future__ import annotations

from typing import Callable

import numpy as np

from .formats import F32, e4m3_table, _nearest_even
from .router import route
from .moe import _silu, _bf16_round

E4M3_MAX = 448.0
_E4M3 = e4m3_table()
_E4M3_POS = _E4M3[:0x7F]          # codes 0..0x7E, increasing


def row_scales(v) -> np.ndarray:
    """s[r] = fp32(amax_r / 448), 1 for an all-zero row.  v: float32 [rows, cols]."""
    v = np.asarray(v, dtype=np.float32)
    amax = np.max(np.abs(v), axis=1) if v.size else np.zeros(v.shape[0], np.float32)
    if not np.all(np.isfinite(amax)):
        raise ValueError("non-finite row")
    s = (amax / F32(E4M3_MAX)).astype(F32)
    return np.where(amax == 0, F32(1.0), s).astype(F32)


def e4m3_encode_signed(q: np.ndarray) -> np.ndarray:
    """Signed E4M3 byte nearest to each finite q (ties to the even code, clamped to +-448)."""
    q = np.asarray(q, dtype=np.float64)
    code = _nearest_even(np.abs(q), _E4M3_POS).astype(np.uint8)
    return np.where(np.signbit(q), code | np.uint8(0x80), code).astype(np.uint8)


def quantize_rows(v):
    """Per-row FP8 quantisation: (codes uint8 [rows, cols], scales float32 [rows])."""
    v = np.asarray(v, dtype=np.float32)
    s = row_scales(v)
    q = (v / s[:, None]).astype(F32)                      # one IEEE division each
    return e4m3_encode_signed(q), s


def dequantize_rows(codes, s) -> np.ndarray:
    """FP64 values E4M3[c] * s[row] (exact)."""
    return _E4M3[np.asarray(codes, dtype=np.int64)] * np.asarray(s, dtype=np.float64)[:, None]


class Fp8Tensor:
    """A weight matrix quantised per output channel (row)."""

    def __init__(self, w):
        self.codes, self.scales = quantize_rows(w)

    def dequant(self) -> np.ndarray:
        return dequantize_rows(self.codes, self.scales)


def expert_mlp_fp8(xhat: np.ndarray, gate: Fp8Tensor, up: Fp8Tensor, down: Fp8Tensor) -> dict:
    """One expert on dequantised FP8 inputs xhat [n, H] (FP64): h rounded to FP32, quantised per
    row, then the down projection."""
    gv = xhat @ gate.dequant().T
    uv = xhat @ up.dequant().T
    h = (_silu(gv) * uv).astype(np.float32)
    hq, hs = quantize_rows(h)
    y = dequantize_rows(hq, hs) @ down.dequant().T
    return {"h": h, "hq_codes": hq, "hq_scales": hs, "y": y}


def moe_forward_fp8(x, w_router, cfg, experts: Callable[[int], tuple], bias=None, tokens=None) -> dict:
    """The FP8 layer: routing as the NVFP4 layer, x quantised per token, experts(e) returns the
    (gate, up, down) Fp8Tensors of expert e."""
    x = np.asarray(x, dtype=np.float32)
    T = x.shape[0]
    r = route(x, w_router, cfg, bias)
    xq, xs = quantize_rows(x)
    tokens = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    out = np.zeros((len(tokens), x.shape[1]), dtype=np.float64)
    need = {}
    for i, t in enumerate(tokens):
        for j in range(cfg.topk):
            need.setdefault(int(r.idx[t, j]), []).append((i, int(t), j))
    for e in sorted(need):
        rows = need[e]
        ts = np.array([t for _, t, _ in rows])
        res = expert_mlp_fp8(dequantize_rows(xq[ts], xs[ts]), *experts(e))
        for n, (i, t, j) in enumerate(rows):
            out[i] += r.w[t, j] * res["y"][n]
    return {"route": r, "xq_codes": xq, "xq_scales": xs, "tokens": tokens, "out": out,
            "out_bf16": _bf16_round(out)}
