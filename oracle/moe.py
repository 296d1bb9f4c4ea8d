"""Expert grouping and the SwiGLU expert MLP on dequantised NVFP4 operands, in FP64.  TEST INFRASTRUCTURE ONLY.

Follows "Reflection releases Beam ...", section "Mixture-of-Experts details"
(each expert is a SwiGLU MLP of intermediate size 2560; only the 8 routed
experts run per token; the expert outputs are combined with the normalised
router weights times 2.5) and "NVFP4 quantization", section "Quantization
scheme" (the expert gate, up and down projections and their input activations
are NVFP4).

Readings where the pages are silent:

* The layer input x is quantised with a dynamic global scale taken from its own
  amax (one tensor: all tokens of the call).
* The intermediate activation h = silu(gate) * up, the input of the down
  projection, is quantised with a static per-expert global scale g_h[e] given
  with the expert (a calibrated constant, as post-training quantisation
  provides), by the same block rule; h is rounded to FP32 first (the SwiGLU
  product is an FP32 quantity on the pages).
* Each of gate, up and down carries its own global scale.
* out[t] = sum over the token's selected experts of w * y, returned in FP64 and
  rounded to BF16 (round-to-nearest-even) as the layer output.
* Grouping: the token/slot pairs are ordered by expert with a stable sort, so
  inside one expert the tokens stay in ascending order.
"""
from __future__ import annotations

import dataclasses
from typing import Callable

import numpy as np

from .formats import quantize, dequantize
from .router import route


@dataclasses.dataclass
class QuantTensor:
    codes: np.ndarray    # uint8 [rows, cols/2]
    scales: np.ndarray   # uint8 [rows, cols/16] linear
    g: np.float32

    def dequant(self) -> np.ndarray:
        return dequantize(self.codes, self.scales, self.g)


def quantize_tensor(x32) -> QuantTensor:
    codes, scales, g = quantize(np.asarray(x32, dtype=np.float32))
    return QuantTensor(codes, scales, g)


def permutation(idx: np.ndarray, E: int):
    """Stable grouping of (token, slot) pairs by expert.

    Pair id p = t * k + j.  Returns counts [E], offsets [E+1] (exclusive scan),
    perm [T*k] (pair ids grouped by expert, ascending inside an expert) and
    inv [T, k] (position of each pair in perm).
    """
    idx = np.asarray(idx, dtype=np.int64)
    T, k = idx.shape
    flat = idx.reshape(-1)
    counts = np.bincount(flat, minlength=E).astype(np.int64)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    perm = np.argsort(flat, kind="stable").astype(np.int64)
    inv = np.empty(T * k, dtype=np.int64)
    inv[perm] = np.arange(T * k)
    return counts, offsets, perm, inv.reshape(T, k)


def _silu(v):
    return v / (1.0 + np.exp(-v))


def expert_mlp(xhat: np.ndarray, gate: QuantTensor, up: QuantTensor, down: QuantTensor,
               g_h) -> dict:
    """One expert on already-dequantised inputs xhat [n, H] (FP64).

    Returns h (FP64), its NVFP4 requantisation (codes, linear scales) and y [n, H].
    """
    Wg = gate.dequant()
    Wu = up.dequant()
    gv = xhat @ Wg.T
    uv = xhat @ Wu.T
    del Wg, Wu
    h = _silu(gv) * uv
    hq_codes, hq_scales, _ = quantize(h.astype(np.float32), g=g_h)
    hhat = dequantize(hq_codes, hq_scales, g_h)
    y = hhat @ down.dequant().T
    return {"gate": gv, "up": uv, "h": h, "hq_codes": hq_codes, "hq_scales": hq_scales, "y": y}


def _bf16_round(v: np.ndarray) -> np.ndarray:
    """Round FP64 values to BF16 (round-to-nearest-even via FP32; exact double rounding
    is avoided by rounding the FP64 value straight to 8 significant bits)."""
    v = np.asarray(v, dtype=np.float64)
    m, e = np.frexp(v)                      # v = m * 2**e, 0.5 <= |m| < 1
    scaled = np.ldexp(m, 8)                 # 8 significant bits -> integer part
    r = np.round(scaled)                    # numpy rounds half to even
    return np.ldexp(r, e - 8)


def moe_forward(x, w_router, cfg, experts: Callable[[int], tuple], g_h, bias=None,
                tokens=None, keep_intermediates: bool = False) -> dict:
    """The routed-expert layer.

    x: [T, H] BF16 values (float32 array); w_router: [E, H]; experts(e) returns
    (gate, up, down) QuantTensors of expert e; g_h: [E] static intermediate
    global scales.  ``tokens``: indices of the tokens whose output is computed
    (default all); routing always covers every token (the global activation
    scale depends on all of x).
    """
    x = np.asarray(x, dtype=np.float32)
    T = x.shape[0]
    r = route(x, w_router, cfg, bias)
    xq_codes, xq_scales, g_x = quantize(x)
    tokens = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    out = np.zeros((len(tokens), x.shape[1]), dtype=np.float64)
    inter = {}
    need = {}
    for i, t in enumerate(tokens):
        for j in range(cfg.topk):
            need.setdefault(int(r.idx[t, j]), []).append((i, int(t), j))
    for e in sorted(need):
        rows = need[e]
        ts = np.array([t for _, t, _ in rows])
        xhat = dequantize(xq_codes[ts], xq_scales[ts], g_x)
        gate, up, down = experts(e)
        res = expert_mlp(xhat, gate, up, down, np.float32(g_h[e]))
        for n, (i, t, j) in enumerate(rows):
            out[i] += r.w[t, j] * res["y"][n]
            if keep_intermediates:
                inter[(t, j)] = {k: res[k][n] for k in ("h", "hq_codes", "hq_scales", "gate", "up")}
    return {"route": r, "xq_codes": xq_codes, "xq_scales": xq_scales, "g_x": g_x,
            "tokens": tokens, "out": out, "out_bf16": _bf16_round(out), "inter": inter}
