"""Local-Hessian block-scale search for NVFP4 weight quantisation.  TEST INFRASTRUCTURE ONLY.

Follows "NVFP4 quantization", section "Quantization method": post-training quantisation in
which, for each block, candidate scales are searched and the one that minimises the
Hessian-weighted error dW^T H dW is kept, H computed from the tokens routed to the expert.

Readings where the page is silent:

* "Local": each 16-value block of a weight row is searched on its own, with H_b, the 16x16
  diagonal block of H = X^T X for the block's 16 input columns (X: calibration inputs of the
  projection, one row per token).  H_b is shared by every row of the weight matrix.
* Candidates: the E4M3 codes S0 - m .. S0 + m, clamped to 1 .. 0x7E, where S0 is the scale
  the round-to-nearest rule of ``formats.quantize`` picks; a block whose amax is 0 keeps 0.
* For a candidate S the codes follow that rule with S_b = S (same global scale g):
  d = fp32(E4M3(S) * g), r_b = fp32(1 / d), c = E2M1(fp32(w * r_b)).
* e(S) = dW^T H_b dW with dW = E2M1(c) * d - w, in FP64.
* Candidates are visited in the order S0, S0-1, S0+1, S0-2, S0+2, ...; one replaces the best so
  far only when its error is strictly smaller (ties keep the scale nearest S0, then the lower).
* The global scale is the rule's g = fp32(A / 2688) of the whole matrix.
"""
from __future__ import annotations

import numpy as np

from .formats import F32, e4m3_encode, e4m3_decode, e2m1_encode, e2m1_decode, global_scale

E4M3_MAX_CODE = 0x7E


def candidate_offsets(m: int) -> list[int]:
    """Visiting order of the code offsets: 0, -1, +1, -2, +2, ..., -m, +m."""
    out = [0]
    for j in range(1, m + 1):
        out += [-j, j]
    return out


def codes_for_scale(wb: np.ndarray, S: np.ndarray, g) -> np.ndarray:
    """E2M1 codes [..., 16] of blocks wb [..., 16] (float32) with block scale codes S [...]."""
    g = F32(g)
    d = (e4m3_decode(S).astype(F32) * g).astype(F32)
    with np.errstate(divide="ignore"):
        r_b = np.where(d == 0, F32(0.0), F32(1.0) / d).astype(F32)
    return e2m1_encode((wb * r_b[..., None]).astype(F32))


def block_error(wb: np.ndarray, c: np.ndarray, S: np.ndarray, g, Hb: np.ndarray) -> np.ndarray:
    """e = dW^T H_b dW per block, FP64: wb [rows, nb, 16], c codes, S [rows, nb], Hb [nb, 16, 16]."""
    d = e4m3_decode(S) * np.float64(F32(g))       # the FP32 d of the rule, exactly
    dw = e2m1_decode(c) * d[..., None] - np.asarray(wb, dtype=np.float64)
    return np.einsum("rbi,bij,rbj->rb", dw, np.asarray(Hb, dtype=np.float64), dw)


def quantize_local_hessian(w, Hb, m: int = 4, g=None):
    """Quantise a [rows, cols] float32 weight matrix with the block-scale search.

    Hb: [cols/16, 16, 16] local Hessian blocks.  Returns (codes uint8 [rows, cols/2],
    scales uint8 [rows, cols/16] linear, g float32, errors FP64 [rows, cols/16, 2m+1] in the
    visiting order, candidate codes [rows, cols/16, 2m+1])."""
    w = np.asarray(w)
    if w.dtype != np.float32:
        raise TypeError("weights must be float32 values (BF16 widens exactly)")
    rows, cols = w.shape
    nb = cols // 16
    if g is None:
        g = global_scale(np.max(np.abs(w)) if w.size else 0.0)
    g = F32(g)
    r_t = F32(1.0) / (F32(6.0) * g)
    wb = w.reshape(rows, nb, 16)
    S0 = e4m3_encode((np.max(np.abs(wb), axis=2) * r_t).astype(F32)).astype(np.int64)
    offs = candidate_offsets(m)
    cands = np.empty((rows, nb, len(offs)), dtype=np.int64)
    errs = np.empty((rows, nb, len(offs)), dtype=np.float64)
    for k, o in enumerate(offs):
        S = np.where(S0 == 0, 0, np.clip(S0 + o, 1, E4M3_MAX_CODE))
        c = codes_for_scale(wb, S.astype(np.uint8), g)
        cands[..., k] = S
        errs[..., k] = block_error(wb, c, S.astype(np.uint8), g, Hb)
    best = np.zeros((rows, nb), dtype=np.int64)
    for k in range(1, len(offs)):
        better = errs[..., k] < np.take_along_axis(errs, best[..., None], axis=2)[..., 0]
        best = np.where(better, k, best)
    S = np.take_along_axis(cands, best[..., None], axis=2)[..., 0].astype(np.uint8)
    c = codes_for_scale(wb, S, g).reshape(rows, cols)
    codes = (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)
    return codes, S, g, errs, cands


def hessian_blocks(x) -> np.ndarray:
    """The 16x16 diagonal blocks of H = X^T X (FP64) for calibration inputs X [n, cols]."""
    x = np.asarray(x, dtype=np.float64)
    n, cols = x.shape
    xb = x.reshape(n, cols // 16, 16)
    return np.einsum("nbi,nbj->bij", xb, xb)
