"""Planted mistakes in the oracle, on the CPU: the pins must notice each one.

Every case below rewrites one expression of one oracle function, in memory only, into a
plausible error (a dropped factor, a wrong sign, index or tie rule, exchanged operands, a
transposed layout) and runs the oracle's pins (``tests/test_oracle_*.py``) against the
planted oracle.  The case passes when some pin fails; a mistake that every pin lets through
fails the case.  The oracle's files are never modified: the planted function is compiled
from the original's source with the one expression replaced, bound in place of the original
wherever the oracle or the pins hold it, and the originals are restored afterwards.
"""
from __future__ import annotations

import __future__
import contextlib
import importlib
import inspect
import sys
import textwrap

import numpy as np
import pytest

PIN_MODULES = {
    "formats": "tests.test_oracle_formats",
    "router": "tests.test_oracle_router",
    "moe": "tests.test_oracle_moe",
    "fp8": "tests.test_oracle_fp8",
    "residual": "tests.test_oracle_residual",
    "local_hessian": "tests.test_oracle_local_hessian",
}


def _pins(first: str):
    """(name, function, kwargs) of every pin, the planted module's own pin file first."""
    order = [PIN_MODULES[first]] + [m for k, m in PIN_MODULES.items() if k != first]
    for mod_name in order:
        mod = importlib.import_module(mod_name)
        for attr, fn in list(vars(mod).items()):
            if not (attr.startswith("test_") and callable(fn)):
                continue
            marks = [m for m in getattr(fn, "pytestmark", []) if m.name == "parametrize"]
            if not marks:
                yield f"{mod_name}::{attr}", fn, {}
                continue
            assert len(marks) == 1, f"{attr}: one parametrize mark expected"
            names = marks[0].args[0]
            names = [n.strip() for n in names.split(",")] if isinstance(names, str) else list(names)
            for vals in marks[0].args[1]:
                vals = tuple(vals) if len(names) > 1 else (vals,)
                yield f"{mod_name}::{attr}{list(vals)}", fn, dict(zip(names, vals))


def _holders():
    """Modules that may hold a reference to an oracle function: the oracle's and the tests'."""
    return [m for n, m in list(sys.modules.items())
            if m is not None and (n == "oracle" or n.startswith(("oracle.", "tests.", "test_oracle")))]


@contextlib.contextmanager
def planted(module: str, func: str, old: str, new: str):
    mod = importlib.import_module(f"oracle.{module}")
    orig = getattr(mod, func)
    src = textwrap.dedent(inspect.getsource(orig))
    assert src.count(old) == 1, f"oracle.{module}.{func}: the expression to plant over is not in its source"
    code = compile(src.replace(old, new), f"<planted oracle.{module}.{func}>", "exec",
                   flags=__future__.annotations.compiler_flag, dont_inherit=True)
    scope: dict = {}
    exec(code, mod.__dict__, scope)
    mutant = scope[func]
    for name in PIN_MODULES.values():
        importlib.import_module(name)
    bound = []
    try:
        for m in _holders():
            for k, v in list(vars(m).items()):
                if v is orig:
                    setattr(m, k, mutant)
                    bound.append((m, k))
        assert bound, "the planted function was bound nowhere"
        yield
    finally:
        for m, k in bound:
            setattr(m, k, orig)


def _first_failing_pin(first: str):
    for name, fn, kw in _pins(first):
        try:
            with np.errstate(all="ignore"):
                fn(**kw)
        except Exception as exc:          # an assertion, or any error the mistake provokes
            return name, exc
    return None


# (id, oracle module, function, expression, planted mistake)
CASES = [
    # formats: the quantisation rule, the number formats, the scale layout, sizes
    ("global-scale-drops-6", "formats", "global_scale",
     "F32(a / F32(2688.0))", "F32(a / F32(448.0))"),
    ("r_t-drops-6", "formats", "quantize",
     "r_t = F32(1.0) / (F32(6.0) * g)", "r_t = F32(1.0) / g"),
    ("block-decode-drops-g", "formats", "quantize",
     "d = (e4m3_decode(S).astype(F32) * g).astype(F32)", "d = e4m3_decode(S).astype(F32)"),
    ("blocks-strided", "formats", "quantize",
     "xb = x.reshape(rows, cols // 16, 16)", "xb = x.reshape(rows, 16, cols // 16).transpose(0, 2, 1)"),
    ("nibbles-swapped", "formats", "quantize",
     "(c[:, 0::2] | (c[:, 1::2] << 4))", "(c[:, 1::2] | (c[:, 0::2] << 4))"),
    ("e2m1-ties-away", "formats", "e2m1_encode",
     "code += (mag > mid) if i % 2 == 0 else (mag >= mid)", "code += (mag >= mid)"),
    ("e2m1-ties-toward-zero", "formats", "e2m1_encode",
     "code += (mag > mid) if i % 2 == 0 else (mag >= mid)", "code += (mag > mid)"),
    ("e2m1-loses-negative-zero", "formats", "e2m1_encode",
     "code[np.signbit(v)] |= np.uint8(8)", "code[v < 0] |= np.uint8(8)"),
    ("e4m3-ties-down", "formats", "_nearest_even",
     "np.where(tie, np.where(lo % 2 == 0, lo, hi), pick)", "np.where(tie, lo, pick)"),
    ("e4m3-ties-odd", "formats", "_nearest_even",
     "np.where(lo % 2 == 0, lo, hi)", "np.where(lo % 2 == 1, lo, hi)"),
    ("swizzle-strides-exchanged", "formats", "swizzle_scales",
     "(r % 32) * 16 + (r % 128 // 32) * 4", "(r % 32) * 4 + (r % 128 // 32) * 16"),
    ("swizzle-row-tile-stride", "formats", "swizzle_scales",
     "(r // 128) * (n_ct * 512)", "(r // 128) * 512"),
    ("dequant-scales-tiled", "formats", "dequantize",
     "np.repeat(s, 16, axis=1)", "np.tile(s, (1, 16))"),
    ("unpack-nibbles-swapped", "formats", "unpack_codes",
     "out[:, 0::2] = codes & 0xF\n    out[:, 1::2] = codes >> 4",
     "out[:, 0::2] = codes >> 4\n    out[:, 1::2] = codes & 0xF"),
    ("swizzle-column-tile-stride", "formats", "swizzle_scales",
     "(c // 4) * 512 + (r % 32)", "(c // 4) * 128 + (r % 32)"),
    ("scale-per-row", "formats", "quantize",
     "amax_b = np.max(np.abs(xb), axis=2) if x.size",
     "amax_b = np.repeat(np.max(np.abs(xb), axis=(1, 2))[:, None], cols // 16, axis=1) if x.size"),
    ("zero-tensor-scale-zero", "formats", "global_scale", "if a == 0:\n        return F32(1.0)",
     "if a == 0:\n        return F32(0.0)"),
    ("e2m1-rounds-down", "formats", "e2m1_encode",
     "mid = (_E2M1_MAG[i] + _E2M1_MAG[i + 1]) / 2", "mid = _E2M1_MAG[i + 1]"),
    ("scale-from-first-value", "formats", "quantize",
     "amax_b = np.max(np.abs(xb), axis=2) if x.size", "amax_b = np.abs(xb[:, :, 0]) if x.size"),
    ("scale-bytes-per-32", "formats", "nvfp4_tensor_bytes",
     "rows * cols // 16", "rows * cols // 32"),
    # router
    ("sigmoid-sign", "router", "_sigmoid", "np.exp(-l)", "np.exp(l)"),
    ("group-score-top1", "router", "route", "[:, :, : min(2, gs)]", "[:, :, : min(1, gs)]"),
    ("group-score-top3", "router", "route", "[:, :, : min(2, gs)]", "[:, :, : min(3, gs)]"),
    ("group-ties-high", "router", "route",
     "np.lexsort((gidx, -gscore[t]))", "np.lexsort((-gidx, -gscore[t]))"),
    ("groups-interleaved", "router", "route",
     "admissible = (eidx // gs)[None, :]", "admissible = (eidx % G)[None, :]"),
    ("one-group-too-few", "router", "route", "kept = np.sort(gorder[:KG])", "kept = np.sort(gorder[:KG - 1])"),
    ("expert-ties-high", "router", "route",
     "cand[np.lexsort((cand, -s[t, cand]))]", "cand[np.lexsort((-cand, -s[t, cand]))]"),
    ("weights-over-all-experts", "router", "route",
     "cfg.routed_scale * ss / ss.sum()", "cfg.routed_scale * ss / s[t].sum()"),
    ("routed-scale-dropped", "router", "route", "cfg.routed_scale * ss / ss.sum()", "ss / ss.sum()"),
    ("weights-not-normalised", "router", "route", "cfg.routed_scale * ss / ss.sum()", "cfg.routed_scale * ss"),
    ("selection-in-index-order", "router", "route", "idx[t] = sel", "idx[t] = np.sort(sel)"),
    ("bias-after-sigmoid", "router", "route",
     "logits = logits + np.asarray(bias, dtype=np.float64)[None, :]",
     "logits = _sigmoid(logits) + np.asarray(bias, dtype=np.float64)[None, :]"),
    ("group-margin-wrong-neighbour", "router", "route",
     "gscore[t, gorder[KG - 1]] - gscore[t, gorder[KG]]", "gscore[t, gorder[0]] - gscore[t, gorder[KG]]"),
    ("expert-margin-off-by-one", "router", "route",
     "s[t, corder[K - 1]] - s[t, corder[K]]", "s[t, corder[K - 2]] - s[t, corder[K]]"),
    ("order-margin-max", "router", "route", "np.min(ss[:-1] - ss[1:])", "np.max(ss[:-1] - ss[1:])"),
    # grouping, expert MLP, combine
    ("inverse-permutation-forward", "moe", "permutation",
     "inv[perm] = np.arange(T * k)", "inv[np.arange(T * k)] = perm"),
    ("tokens-descending-in-expert", "moe", "permutation",
     'perm = np.argsort(flat, kind="stable")', 'perm = flat.size - 1 - np.argsort(flat[::-1], kind="stable")'),
    ("offsets-inclusive", "moe", "permutation", "offsets[1:] = np.cumsum(counts)", "offsets[:-1] = np.cumsum(counts)"),
    ("swiglu-operands-exchanged", "moe", "expert_mlp", "h = _silu(gv) * uv", "h = _silu(uv) * gv"),
    ("silu-drops-v", "moe", "_silu", "v / (1.0 + np.exp(-v))", "1.0 / (1.0 + np.exp(-v))"),
    ("down-on-unquantised-h", "moe", "expert_mlp", "y = hhat @ down.dequant().T", "y = h @ down.dequant().T"),
    ("combine-first-slot-weight", "moe", "moe_forward", "out[i] += r.w[t, j] *", "out[i] += r.w[t, 0] *"),
    ("gather-by-output-index", "moe", "moe_forward",
     "ts = np.array([t for _, t, _ in rows])", "ts = np.array([i for i, _, _ in rows])"),
    ("input-not-quantised", "moe", "moe_forward",
     "xhat = dequantize(xq_codes[ts], xq_scales[ts], g_x)", "xhat = x[ts].astype(np.float64)"),
    ("bf16-truncates", "moe", "_bf16_round", "r = np.round(scaled)", "r = np.trunc(scaled)"),
    ("h-dynamic-scale", "moe", "expert_mlp",
     "hq_codes, hq_scales, _ = quantize(h.astype(np.float32), g=g_h)",
     "hq_codes, hq_scales, g_h = quantize(h.astype(np.float32))"),
    ("g_h-of-expert-0", "moe", "moe_forward",
     "res = expert_mlp(xhat, gate, up, down, np.float32(g_h[e]))",
     "res = expert_mlp(xhat, gate, up, down, np.float32(g_h[0]))"),
    ("gate-and-up-both-gate", "moe", "expert_mlp", "uv = xhat @ Wu.T", "uv = xhat @ Wg.T"),
    ("counts-shifted", "moe", "permutation",
     "counts = np.bincount(flat, minlength=E).astype(np.int64)",
     "counts = np.roll(np.bincount(flat, minlength=E).astype(np.int64), 1)"),
    ("combine-unweighted", "moe", "moe_forward", "out[i] += r.w[t, j] * res[\"y\"][n]", "out[i] += res[\"y\"][n]"),
    ("weights-of-expert-0", "moe", "moe_forward", "gate, up, down = experts(e)", "gate, up, down = experts(0)"),
    # FP8 variant
    ("fp8-fnuz-max", "fp8", "row_scales", "(amax / F32(E4M3_MAX))", "(amax / F32(240.0))"),
    ("fp8-zero-row-scale", "fp8", "row_scales", "np.where(amax == 0, F32(1.0), s)", "s"),
    ("fp8-per-tensor-scale", "fp8", "quantize_rows",
     "s = row_scales(v)", "s = np.full(v.shape[0], row_scales(v).max(), dtype=F32)"),
    ("fp8-reciprocal-multiply", "fp8", "quantize_rows",
     "q = (v / s[:, None]).astype(F32)", "q = (v * (F32(1.0) / s)[:, None]).astype(F32)"),
    ("fp8-loses-negative-zero", "fp8", "e4m3_encode_signed", "np.where(np.signbit(q),", "np.where(q < 0,"),
    ("fp8-swiglu-exchanged", "fp8", "expert_mlp_fp8", "h = (_silu(gv) * uv)", "h = (_silu(uv) * gv)"),
    ("fp8-down-on-unquantised-h", "fp8", "expert_mlp_fp8",
     "y = dequantize_rows(hq, hs) @ down.dequant().T", "y = h.astype(np.float64) @ down.dequant().T"),
    ("fp8-combine-first-slot-weight", "fp8", "moe_forward_fp8", "out[i] += r.w[t, j] *", "out[i] += r.w[t, 0] *"),
    ("fp8-input-not-quantised", "fp8", "moe_forward_fp8",
     "res = expert_mlp_fp8(dequantize_rows(xq[ts], xs[ts]), *experts(e))",
     "res = expert_mlp_fp8(x[ts].astype(np.float64), *experts(e))"),
    # residual stream neighbours
    ("residual-weights-exchanged", "residual", "residual_weights",
     "return np.float32(np.sqrt((k - 1) / k)), np.float32(1.0 / np.sqrt(k))",
     "return np.float32(1.0 / np.sqrt(k)), np.float32(np.sqrt((k - 1) / k))"),
    ("rms-sum-not-mean", "residual", "rmsnorm_scale", "np.mean(h * h, axis=1)", "np.sum(h * h, axis=1)"),
    ("rms-eps-outside-root", "residual", "rmsnorm_scale",
     "1.0 / np.sqrt(ms + float(eps))", "1.0 / (np.sqrt(ms) + float(eps))"),
    ("rms-divides", "residual", "rmsnorm", "(h32 * r[:, None])", "(h32 / r[:, None])"),
    ("rms-gamma-dropped", "residual", "rmsnorm",
     "(y * np.asarray(gamma, dtype=np.float32)[None, :])", "(y * np.float32(1.0))"),
    ("residual-add-exchanged", "residual", "residual_add",
     "float(a) * np.asarray(h, dtype=np.float64) + float(b) * np.asarray(moe_out, dtype=np.float64)",
     "float(b) * np.asarray(h, dtype=np.float64) + float(a) * np.asarray(moe_out, dtype=np.float64)"),
    # local-Hessian scale search
    ("lh-order-plus-first", "local_hessian", "candidate_offsets", "out += [-j, j]", "out += [j, -j]"),
    ("lh-ties-to-later", "local_hessian", "quantize_local_hessian",
     "better = errs[..., k] <", "better = errs[..., k] <="),
    ("lh-codes-drop-g", "local_hessian", "codes_for_scale",
     "d = (e4m3_decode(S).astype(F32) * g).astype(F32)", "d = e4m3_decode(S).astype(F32)"),
    ("lh-error-unweighted", "local_hessian", "block_error",
     'np.einsum("rbi,bij,rbj->rb", dw, np.asarray(Hb, dtype=np.float64), dw)', 'np.einsum("rbi,rbi->rb", dw, dw)'),
    ("lh-hessian-strided", "local_hessian", "hessian_blocks",
     "xb = x.reshape(n, cols // 16, 16)", "xb = x.reshape(n, 16, cols // 16).transpose(0, 2, 1)"),
    ("lh-window-one-sided", "local_hessian", "quantize_local_hessian",
     "np.clip(S0 + o, 1, E4M3_MAX_CODE)", "np.clip(S0 + abs(o), 1, E4M3_MAX_CODE)"),
]


def test_pins_pass_without_a_planted_mistake():
    """The harness runs the pins as the test run does: with nothing planted, none fails."""
    assert _first_failing_pin("formats") is None


@pytest.mark.parametrize("module,func,old,new", [c[1:] for c in CASES], ids=[c[0] for c in CASES])
def test_planted_mistake_is_caught(module, func, old, new):
    with planted(module, func, old, new):
        caught = _first_failing_pin(module)
    assert caught is not None, f"no pin notices oracle.{module}.{func}: {old!r} -> {new!r}"
