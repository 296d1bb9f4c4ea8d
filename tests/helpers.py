"""Shared test plumbing: oracle-side layer construction, the router near-tie protocol and
output tolerances.  Oracle calls only: nothing here reads a value computed by the CUDA
library except the GPU results under test, which are only compared."""
from __future__ import annotations

import math
import multiprocessing as mp
import os
import types

import numpy as np
import torch

import oracle
from workloads import TINY, BEAM, activations, router_weight, expert_weight, zipf_bias
from tests.conftest import read_golden

U = 2.0 ** -24


def cfg_ns(shape):
    return types.SimpleNamespace(E=shape.E, n_groups=shape.n_groups, topk_groups=shape.topk_groups,
                                 topk=shape.topk, routed_scale=shape.routed_scale)


def intermediate_scales(shape) -> np.ndarray:
    """Static g_h[e] of the layer, as written by tests/golden/make_intermediate_scales.py."""
    name = {TINY: "tiny", BEAM: "beam"}[shape]
    rows = read_golden(f"intermediate_scales_{name}.txt")
    g = np.array([int(h, 16) for _, h, _ in rows], dtype=np.uint32).view(np.float32)
    assert len(g) == shape.E
    return g


# ------------------------------------------------------------------ router ----

def _row_exponents(v: np.ndarray) -> np.ndarray:
    """Per row, the binary exponent e with max|v| < 2^e, at least -125 (the library's rule:
    rows whose maximum is zero or subnormal take the smallest normal exponent)."""
    m = np.max(np.abs(v), axis=1)
    e = np.frexp(m)[1].astype(np.int64)
    return np.where(m == 0, -125, np.maximum(e, -125))


def _fixed_point(v: np.ndarray, bits: int) -> np.ndarray:
    """Each row scaled to `bits`-bit fixed point from its exponent and rounded to the nearest
    integer (ties to even), in the row's own units: RNE(v 2^(bits - e)) 2^(e - bits)."""
    e = _row_exponents(v)[:, None]
    return np.ldexp(np.rint(np.ldexp(v, bits - e)), e - bits)


def router_logit_bound_int(x: np.ndarray, wr: np.ndarray, bias, H: int, worst: bool = False) -> np.ndarray:
    """The documented bound of the integer tensor-core logits (T > 64):
    2^-24 |logit| + sum_h |x_h - x'_h| |W_eh| + sum_h |x_h| |W_eh - W'_eh| + H 2^(e_x + e_W - 28),
    x' and W' the 22-bit and 30-bit fixed-point rows the kernel multiplies.  ``worst``: the two
    rounding sums replaced by their worst case 2^(e_x - 23) sum|W_e| + 2^(e_W - 31) sum|x_t|
    (row sums only: cheap at any T)."""
    ex = _row_exponents(x)[:, None].astype(np.float64)
    ew = _row_exponents(wr)[None, :].astype(np.float64)
    logit = x @ wr.T
    if bias is not None:
        logit = logit + np.asarray(bias, dtype=np.float64)[None, :]
    if worst:
        rx = np.exp2(ex - 23) * np.abs(wr).sum(axis=1)[None, :]
        rw = np.exp2(ew - 31) * np.abs(x).sum(axis=1)[:, None]
    else:
        rx = np.abs(x - _fixed_point(x, 22)) @ np.abs(wr).T
        rw = np.abs(x) @ np.abs(wr - _fixed_point(wr, 30)).T
    return U * np.abs(logit) + rx + rw + H * np.exp2(ex + ew - 28) + 2.0 ** -60


def router_logit_bound_fp32(x: np.ndarray, wr: np.ndarray, bias, H: int) -> np.ndarray:
    """The documented bound of the FP32 logits (T <= 64, and the allocation-free router):
    32 * 2^-24 * sum_h |x_h W_eh| + 2^-24 |logit| (FP64 terms covered by a 2^-40 margin)."""
    sabs = np.abs(x) @ np.abs(wr).T
    logit = x @ wr.T
    if bias is not None:
        logit = logit + np.asarray(bias, dtype=np.float64)[None, :]
    return 32 * U * sabs + U * np.abs(logit) + 2.0 ** -40 * (sabs + 1)


def router_logit_bound(x: np.ndarray, wr: np.ndarray, bias, H: int) -> np.ndarray:
    """A bound that holds for either logits path: the larger of the two documented ones (the
    integer one in its worst-case form)."""
    return np.maximum(router_logit_bound_fp32(x, wr, bias, H), router_logit_bound_int(x, wr, bias, H, worst=True))


def check_routing(gpu_idx: np.ndarray, gpu_w: np.ndarray, r, x, wr, bias, shape, w_rtol=2e-6,
                  bound=router_logit_bound):
    """Near-tie protocol.  A token is clean when every routing decision has a margin larger
    than the FP32 error bound; clean tokens must match the oracle bit for bit (experts and
    their order).  Other tokens must pick an admissible selection: experts from groups and
    scores within the error bound of the exact choice.  Weights are compared (relative
    tolerance) against the oracle's weights of the GPU's own selection.  ``bound`` gives the
    logit error bound of the path under test (default: the larger of the two documented ones).
    Returns (clean token mask, number of flagged tokens)."""
    T, K = gpu_idx.shape
    gs = shape.E // shape.n_groups
    bl = bound(x, wr, bias, shape.H)
    s = r.scores
    eps_s = bl * s * (1 - s) + 8 * U                       # sigmoid: Lipschitz s(1-s) + its own rounding
    eps = eps_s.max(axis=1)                                # per token
    dgrp = 2 * eps + 2 * U                                 # error of one group score
    clean = (r.expert_margin > 2 * eps) & (r.group_margin > 2 * dgrp) & (r.order_margin > 2 * eps)
    n_flag = int((~clean).sum())
    # clean tokens: exact
    mism = clean & (gpu_idx != r.idx).any(axis=1)
    assert not mism.any(), f"{int(mism.sum())} clean tokens routed differently, e.g. {np.flatnonzero(mism)[:5]}"
    # every token: a valid, admissible selection
    for t in range(T):
        sel = gpu_idx[t]
        assert len(set(sel.tolist())) == K and sel.min() >= 0 and sel.max() < shape.E
        if clean[t]:
            continue
        kth = np.sort(s[t, r.idx[t]])[0]
        g4 = np.sort(r.group_scores[t])[::-1][shape.topk_groups - 1]
        assert np.all(s[t, sel] >= kth - 2 * eps[t]), f"token {t}: expert score below admissible range"
        assert np.all(r.group_scores[t, sel // gs] >= g4 - 2 * dgrp[t]), f"token {t}: group not admissible"
    # weights of the GPU's selection
    ssel = np.take_along_axis(s, gpu_idx.astype(np.int64), axis=1)
    w_ref = shape.routed_scale * ssel / ssel.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(gpu_w, w_ref, rtol=w_rtol, atol=0)
    return clean, n_flag


# ------------------------------------------------------------------ experts ----

def oracle_expert(shape, e: int, seed: int = 0):
    """Expert e quantised by the oracle from the seeded BF16 weights."""
    return tuple(oracle.quantize_tensor(expert_weight(shape, e, w, seed=seed).float().numpy())
                 for w in ("gate", "up", "down"))


def _abs_sums(xhat, t: "oracle.QuantTensor") -> np.ndarray:
    """sum_k |x_k w_k| of every (row, output) of a product with dequantised operands (the scale of
    the FP32 accumulation error of that output)."""
    return np.abs(xhat) @ np.abs(t.dequant()).T


def accumulation_bound(xhat, t: "oracle.QuantTensor", step: int = 64) -> np.ndarray:
    """Bound on |acc - exact| of every (row, output) of x W^T accumulated as the grouped GEMM
    issues it: K in ascending order, one tensor-core instruction per ``step`` values, each adding
    its exact products into the FP32 accumulator.  Per instruction i at most one rounding of the
    running sum P_i (2^-23 |P_i|) and an internal error of at most 2^-23 sum|products of i|:
    2^-23 (sum_i |P_i| + sum_k |x_k w_k|)."""
    W = t.dequant()
    K = xhat.shape[1]
    P = np.zeros((xhat.shape[0], W.shape[0]))
    total = np.zeros_like(P)
    for k0 in range(0, K, step):
        xs, ws = xhat[:, k0:k0 + step], W[:, k0:k0 + step]
        P += xs @ ws.T
        total += np.abs(P) + np.abs(xs) @ np.abs(ws).T
    return U23 * total


def _expert_job(args):
    shape, e, xhat, g_h = args
    gate, up, down = oracle_expert(shape, e)
    res = oracle.expert_mlp(xhat, gate, up, down, np.float32(g_h))
    dh = h_error_bound(res["gate"], res["up"], accumulation_bound(xhat, gate), accumulation_bound(xhat, up))
    return e, res["y"], res["h"], res["hq_codes"], res["hq_scales"], dh


def _init_single_thread():
    from threadpoolctl import threadpool_limits
    threadpool_limits(limits=1)


def _expert_rows_job(args):
    """One expert on a batch of dequantised input rows (possibly from several layer calls):
    the oracle's SwiGLU MLP and requantised h, plus the down projection of the GPU's own
    requantised h of the same rows (the oracle run on the same quantised operands)."""
    shape, e, xhat, g_h, gpu_hq_codes, gpu_hq_scales = args
    gate, up, down = oracle_expert(shape, e)
    res = oracle.expert_mlp(xhat, gate, up, down, np.float32(g_h))
    y_gpu_hq = res["y"].copy()
    if gpu_hq_codes is None:
        return e, res["y"], y_gpu_hq, res["h"], res["hq_codes"], res["hq_scales"], None
    dh = h_error_bound(res["gate"], res["up"], accumulation_bound(xhat, gate), accumulation_bound(xhat, up))
    same = (np.all(gpu_hq_codes == res["hq_codes"], axis=1) & np.all(gpu_hq_scales == res["hq_scales"], axis=1))
    if not same.all():
        hhat = oracle.dequantize(gpu_hq_codes[~same], gpu_hq_scales[~same], np.float32(g_h))
        y_gpu_hq[~same] = hhat @ down.dequant().T
    return e, res["y"], y_gpu_hq, res["h"], res["hq_codes"], res["hq_scales"], dh


def oracle_expert_pass(shape, jobs: dict, workers=None) -> dict:
    """Runs _expert_rows_job for every expert of ``jobs`` (e -> (xhat, g_h, gpu hq codes,
    gpu hq scales), the last two None when there is no GPU intermediate to reuse) in a spawn
    process pool, one BLAS thread per worker."""
    args = [(shape, e, *v) for e, v in sorted(jobs.items())]
    if workers is None:
        workers = max(1, min(len(args), len(os.sched_getaffinity(0)) - 1))
    if workers > 1:
        with mp.get_context("spawn").Pool(workers, initializer=_init_single_thread) as pool:
            results = pool.map(_expert_rows_job, args, chunksize=1)
    else:
        results = [_expert_rows_job(a) for a in args]
    return {r[0]: r[1:] for r in results}


def oracle_layer(shape, x: np.ndarray, wr: np.ndarray, bias, g_h: np.ndarray, tokens=None, workers=None,
                 expert_range=None):
    """Oracle layer output for the given tokens: routing of all tokens, expert MLPs of the
    sampled tokens (experts evaluated in a spawn process pool when there are many).  With
    expert_range = (first, count) only those experts' contributions are summed (one rank's
    part under expert parallelism)."""
    cfg = cfg_ns(shape)
    r = oracle.route(x, wr, cfg, bias)
    xc, xs, gx = oracle.quantize(np.asarray(x, dtype=np.float32))
    T = x.shape[0]
    tokens = np.arange(T) if tokens is None else np.asarray(tokens)
    need = {}
    for i, t in enumerate(tokens):
        for j in range(cfg.topk):
            e = int(r.idx[t, j])
            if expert_range is None or expert_range[0] <= e < expert_range[0] + expert_range[1]:
                need.setdefault(e, []).append((i, int(t), j))
    jobs = []
    for e, rows in sorted(need.items()):
        ts = np.array([t for _, t, _ in rows])
        jobs.append((shape, e, oracle.dequantize(xc[ts], xs[ts], gx), float(g_h[e])))
    if workers is None:
        workers = min(len(jobs), max(1, len(os.sched_getaffinity(0)) // 2)) if len(jobs) > 8 else 1
    if workers > 1:
        with mp.get_context("spawn").Pool(workers) as pool:
            results = pool.map(_expert_job, jobs)
    else:
        results = [_expert_job(j) for j in jobs]
    out = np.zeros((len(tokens), x.shape[1]))
    inter = {}
    for e, y, h, hc, hs, dh in results:
        for n, (i, t, j) in enumerate(need[e]):
            out[i] += r.w[t, j] * y[n]
            inter[(t, j)] = (h[n], hc[n], hs[n], dh[n])
    return {"route": r, "xq_codes": xc, "xq_scales": xs, "g_x": gx, "tokens": tokens, "out": out,
            "inter": inter}


def bf16_half_ulp(v: np.ndarray) -> np.ndarray:
    """Half a BF16 unit in the last place at |v| (the output format's own rounding)."""
    a = np.maximum(np.abs(v), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 8)


def check_output(gpu_out: np.ndarray, ref: np.ndarray, max_abs=2e-2, rel_fro=5e-3, bf16: bool = False):
    """Layer output tolerance: max-abs 2e-2 and relative Frobenius 5e-3 against the oracle's
    FP64 output.  gpu_out is the layer's FP32 sums, or (bf16=True) its BF16 output, whose own
    rounding is then part of the error: half a BF16 unit in the last place stays below 2e-2
    only for |value| < 8, which such a check requires of every reference value."""
    if bf16:
        assert np.all(np.abs(ref) < 8.0), f"an output of magnitude {np.abs(ref).max():.3g} is beyond the range " \
                                          "where the BF16 rounding alone stays below the limit"
    err = np.abs(gpu_out - ref)
    bad = err > max_abs
    assert not bad.any(), f"{int(bad.sum())} outputs beyond tolerance; worst {err.max():.4g}"
    fro = np.linalg.norm(gpu_out - ref) / max(np.linalg.norm(ref), 1e-30)
    assert fro <= rel_fro, f"relative Frobenius error {fro:.3g}"
    return float(err.max()), float(fro)


E2M1_MIDS = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
U23 = 2.0 ** -23


def h_error_bound(gate: np.ndarray, up: np.ndarray, acc_gate: np.ndarray, acc_up: np.ndarray) -> np.ndarray:
    """Bound on |h_gpu - h| for every element of the SwiGLU product as the gate/up epilogue
    computes it, from the oracle's exact gate and up values and the bounds on their FP32
    accumulation errors (accumulation_bound; the block-scaled products themselves are exact in
    FP32: E2M1 x E2M1 x two E4M3 scales).

    * The global-scale multiply rounds once more: dg = acc_gate + 2^-24 |g| (du alike).
    * h = fl(fl(g u) rcp(fl(1 + e))), e = __expf(-g): __expf within (2 + 1.173 |g|) ulp, entering
      1 / (1 + e) with weight e / (1 + e) = 1 - s(g); the sum, the two products and the
      approximate reciprocal (1 ulp) add 3 2^-24 + 2^-23 relative.
    * Propagation to first order, doubled: dh = 2 (|u| |silu'(g)| dg + |silu(g)| du) + |h| eps_f."""
    g = np.asarray(gate, dtype=np.float64)
    u = np.asarray(up, dtype=np.float64)
    s = 1.0 / (1.0 + np.exp(-g))
    dg = acc_gate + 2.0 ** -24 * np.abs(g)
    du = acc_up + 2.0 ** -24 * np.abs(u)
    dsilu = s * (1.0 + g * (1.0 - s))
    h = g * s * u
    eps_f = 3 * 2.0 ** -24 + U23 + (2.0 + 1.173 * np.abs(g)) * U23 * (1.0 - s)
    return 2.0 * (np.abs(u) * np.abs(dsilu) * dg + np.abs(g * s) * du) + np.abs(h) * eps_f


def requant_near_tie(h: np.ndarray, g_h: float, dh: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Where the requantisation of h (exact, FP64) can round the other way for a value within
    dh (h_error_bound) of it: per block, the E4M3 scale of amax / (6 g_h) lies within the
    propagated bound (plus the FP32 roundings of h and of the scaled amax) of an E4M3
    rounding boundary; per element, the scaled value h / d_b lies within its bound of an E2M1
    boundary, or of zero (the sign of zero: codes 0x0 and 0x8 both decode to zero)."""
    h = np.asarray(h, dtype=np.float64)
    n = h.shape[-1]
    hb = h.reshape(-1, n // 16, 16)
    db = np.asarray(dh, dtype=np.float64).reshape(hb.shape) + 2.0 ** -24 * np.abs(hb)
    r_t = 1.0 / (6.0 * g_h)
    amax = np.abs(hb).max(axis=2)
    q = amax * r_t
    dq = r_t * db.max(axis=2) + 2 * U23 * q
    grid = oracle.e4m3_table()[:127]
    mids = (grid[:-1] + grid[1:]) / 2
    block_tie = np.min(np.abs(q[..., None] - mids[None, None, :]), axis=-1) <= dq
    S = oracle.e4m3_encode(q.astype(np.float32))
    d = oracle.e4m3_decode(S) * g_h
    rb = 1.0 / np.where(d == 0, np.inf, d)[..., None]
    v = np.abs(hb) * rb
    dv = db * rb + 2 * U23 * v
    elem_tie = (np.min(np.abs(v[..., None] - E2M1_MIDS), axis=-1) <= dv) | (v <= dv)
    return block_tie.reshape(h.shape[:-1] + (n // 16,)), elem_tie.reshape(h.shape)


# ------------------------------------------------------------------ FP8 W8A8 ----

def oracle_expert_fp8(shape, e: int, seed: int = 0):
    """Expert e quantised per output channel by the oracle (FP8 W8A8 variant)."""
    return tuple(oracle.fp8.Fp8Tensor(expert_weight(shape, e, w, seed=seed).float().numpy())
                 for w in ("gate", "up", "down"))


def _expert_job_fp8(args):
    shape, e, xhat = args
    return e, oracle.fp8.expert_mlp_fp8(xhat, *oracle_expert_fp8(shape, e))["y"]


def oracle_layer_fp8(shape, x: np.ndarray, wr: np.ndarray, bias, tokens=None, workers=None):
    """oracle.fp8.moe_forward_fp8 for the given tokens, its experts evaluated in a spawn
    process pool when there are many (same steps, same functions)."""
    cfg = cfg_ns(shape)
    r = oracle.route(x, wr, cfg, bias)
    xq, xs = oracle.fp8.quantize_rows(np.asarray(x, dtype=np.float32))
    T = x.shape[0]
    tokens = np.arange(T) if tokens is None else np.asarray(tokens)
    need = {}
    for i, t in enumerate(tokens):
        for j in range(cfg.topk):
            need.setdefault(int(r.idx[t, j]), []).append((i, int(t), j))
    jobs = []
    for e, rows in sorted(need.items()):
        ts = np.array([t for _, t, _ in rows])
        jobs.append((shape, e, oracle.fp8.dequantize_rows(xq[ts], xs[ts])))
    if workers is None:
        workers = min(len(jobs), max(1, len(os.sched_getaffinity(0)) // 2)) if len(jobs) > 8 else 1
    if workers > 1:
        with mp.get_context("spawn").Pool(workers) as pool:
            results = pool.map(_expert_job_fp8, jobs)
    else:
        results = [_expert_job_fp8(j) for j in jobs]
    out = np.zeros((len(tokens), x.shape[1]))
    for e, y in results:
        for n, (i, t, j) in enumerate(need[e]):
            out[i] += r.w[t, j] * y[n]
    return {"route": r, "xq_codes": xq, "xq_scales": xs, "tokens": tokens, "out": out}
