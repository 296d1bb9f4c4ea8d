"""The error bound of the gate/up epilogue (tests.helpers.h_error_bound with
accumulation_bound), checked on the CPU against an FP32 emulation of that epilogue: the exact
block-scaled products summed 64 at a time in ascending K (each 64-product sum rounded once
into an FP32 accumulator, the order the grouped GEMM issues its instructions in), the FP32
global-scale multiply, and the SwiGLU product with float32 operations (exp, the 1 + e sum,
the reciprocal and the two products each rounded once).  Every emulated h must lie within the
bound of the exact FP64 value, and the bound must not be vacuous."""
import numpy as np

import oracle
from workloads import TINY, BEAM, activations
from tests.helpers import oracle_expert, h_error_bound, requant_near_tie, accumulation_bound


def _emulated_h(xhat, gate, up):
    """h as an FP32 epilogue computes it from the same operands (scales folded into the
    dequantised values, so the 'global-scale multiply' is a rounding of the exact product)."""
    Wg, Wu = gate.dequant(), up.dequant()
    K = xhat.shape[1]
    order = range(K // 64)

    def acc(W):
        a = np.zeros((xhat.shape[0], W.shape[0]), dtype=np.float32)
        for b in order:
            part = xhat[:, 64 * b:64 * (b + 1)] @ W[:, 64 * b:64 * (b + 1)].T   # exact in FP64 here
            a = (a + part.astype(np.float32)).astype(np.float32)
        return a

    g = acc(Wg)
    u = acc(Wu)
    e = np.exp(-g).astype(np.float32)
    den = (np.float32(1.0) + e).astype(np.float32)
    return ((g * u).astype(np.float32) * (np.float32(1.0) / den).astype(np.float32)).astype(np.float32)


def _case(shape, e, T, seed):
    x = activations(T, shape, seed=seed).float().numpy()
    xc, xs, gx = oracle.quantize(x)
    xhat = oracle.dequantize(xc, xs, gx)
    gate, up, down = oracle_expert(shape, e)
    res = oracle.expert_mlp(xhat, gate, up, down, np.float32(0.004))
    dh = h_error_bound(res["gate"], res["up"], accumulation_bound(xhat, gate), accumulation_bound(xhat, up))
    return xhat, gate, up, res, dh


def test_emulated_fp32_epilogue_within_the_bound_tiny():
    xhat, gate, up, res, dh = _case(TINY, 3, 64, 5)
    h32 = _emulated_h(xhat, gate, up)
    err = np.abs(h32.astype(np.float64) - res["h"])
    assert np.all(err <= dh), f"max err / bound {np.max(err / dh):.3f}"
    # not vacuous: the bound is within a few hundred FP32 units of the values it covers
    assert np.median(dh / np.maximum(np.abs(res["h"]), 1e-3)) < 1e-4


def test_emulated_fp32_epilogue_within_the_bound_beam_expert():
    xhat, gate, up, res, dh = _case(BEAM, 17, 6, 8)
    h32 = _emulated_h(xhat, gate, up)
    err = np.abs(h32.astype(np.float64) - res["h"])
    assert np.all(err <= dh), f"max err / bound {np.max(err / dh):.3f}"
    assert np.max(err / dh) > 0.02                      # the emulated errors reach into the bound
    assert np.median(dh / np.maximum(np.abs(res["h"]), 1e-3)) < 2e-4


def test_near_tie_band_flags_few_elements():
    """With that bound, a small share of the requantisation decisions counts as a near-tie, and
    a value placed exactly on an E2M1 boundary is flagged."""
    xhat, gate, up, res, dh = _case(BEAM, 17, 6, 8)
    block_tie, elem_tie = requant_near_tie(res["h"], 0.004, dh)
    assert block_tie.mean() < 0.01 and elem_tie.mean() < 0.005
    h = res["h"].copy()
    # put one element of row 0's first block exactly on the 1.25 boundary of its block's scale
    r_t = 1.0 / (6.0 * 0.004)
    q = np.abs(h[0, :16]).max() * r_t
    d = oracle.e4m3_decode(oracle.e4m3_encode(np.array([q], dtype=np.float32)))[0] * 0.004
    k = int(np.argmin(np.abs(h[0, :16])))
    h[0, k] = 1.25 * d
    _, elem = requant_near_tie(h, 0.004, dh)
    assert elem[0, k]
