"""The Beam-shape layer (hidden 5120, 256 experts of intermediate 2560 in 8 groups of 32,
top-4 groups, top-8 experts, x2.5) against the oracle at every token count the kernels treat
differently, with samples chosen to reach every kind of tile the grouped GEMMs run.

Sources: "NVFP4 quantization", section "Quantization scheme" (E2M1 values with an E4M3 scale
per 16 values and an FP32 scale per tensor, for the expert projections and their inputs);
"Reflection releases Beam ...", section "Mixture-of-Experts details" (the router and the
SwiGLU experts and their weighted combine).

Cases: T = 8 and 64 (every token; the fused front end), 512 and 1023 (the last token counts
whose expert segments average fewer than 32 rows, so the GEMMs take their decode epilogues),
1024 (the first with the full-segment epilogues), the 4096-token prefill batch (256 sampled
tokens), 16384 tokens under the Zipf router bias (the heaviest experts take thousands of rows,
the lightest a few dozen), 2048 tokens under three times that bias (179 experts receive no
token, 13 one or two, the heaviest about 2000: empty and one-row segments under the
full-segment epilogues) and 32768 tokens.  Sampled tokens are picked from the oracle's own
grouping: the rows that open the second and later 128-row tiles of the heaviest experts'
segments, the last row of those segments (their last, partial tile), every row of experts
holding one or two rows, and seeded random tokens.

For every case: routing of all tokens under the near-tie protocol; the input's global scale,
codes and scales bit-exact; the grouping exactly the oracle's stable sort of the GPU routing;
the FP32 SwiGLU product of every sampled pair (exported by the epilogue) within the derived
error bound of that epilogue (h_error_bound) of the exact value, and its requantisation equal
to the oracle's except where the exact value lies within that bound of a rounding boundary; the FP32 sums of the sampled tokens within max-abs 2e-2 and
relative Frobenius 5e-3 of the oracle run on the same quantised operands (the GPU's own
requantised intermediate, where it differs at a near-tie), the fully independent oracle
output reported beside it, and the BF16 output exactly the round-to-nearest-even of the FP32
sums (so the output's own rounding is checked by its definition, not inside the tolerance:
half a BF16 unit exceeds 2e-2 once |value| >= 8, which the strongly biased case reaches).  The oracle evaluates each expert once for all cases (a spawn
process pool)."""
from __future__ import annotations

import dataclasses

import numpy as np
import pytest
import torch

import oracle
import nvfp4_quantized_moe_group_b200 as moe
from workloads import BEAM, activations, router_weight, zipf_bias
from tests.helpers import (cfg_ns, check_routing, intermediate_scales, check_output, requant_near_tie,
                           oracle_expert_pass)
from tests.test_gpu_forward import gpu_experts, check_grouping

pytestmark = pytest.mark.gpu


@dataclasses.dataclass(frozen=True)
class Case:
    name: str
    T: int
    n_sample: int          # tokens whose outputs are checked (all when >= T)
    seed: int = 0
    bias_scale: float = 0.0   # router logit bias: this multiple of the Zipf bias (0: none)
    n_heavy: int = 16      # heaviest experts whose later tiles are sampled
    tiles_each: int = 3    # tile starts sampled per heavy expert (after the first tile)


CASES = [
    Case("T8", 8, 8, seed=21),
    Case("T64", 64, 64, seed=22),
    Case("T512", 512, 48, seed=23),
    Case("T1023", 1023, 48, seed=24),
    Case("T1024", 1024, 48, seed=25),
    Case("prefill_T4096", 4096, 256, seed=0, n_heavy=32),
    Case("skewed_T16384", 16384, 160, seed=0, bias_scale=1.0, n_heavy=3, tiles_each=6),
    Case("strong_skew_T2048", 2048, 96, seed=27, bias_scale=3.0, n_heavy=4, tiles_each=4),
    Case("T32768", 32768, 96, seed=26, n_heavy=16, tiles_each=4),
]


def pick_tokens(case: Case, r) -> np.ndarray:
    """Sampled tokens, from the oracle's grouping of the oracle's routing."""
    T, k = r.idx.shape
    if case.n_sample >= T:
        return np.arange(T)
    counts, offsets, perm, _ = oracle.permutation(r.idx, BEAM.E)
    chosen: list[int] = []

    def add(row_of_expert, e):
        t = int(perm[offsets[e] + row_of_expert]) // k
        if t not in chosen:
            chosen.append(t)

    heavy = np.argsort(-counts, kind="stable")[:case.n_heavy]
    for e in heavy:
        c = int(counts[e])
        starts = list(range(128, c, 128))
        # the second tile, then the last tiles of the segment
        picks = starts[:1] + starts[1:][-(case.tiles_each - 1):] if case.tiles_each > 1 else starts[:1]
        for row in picks + [c - 1]:
            add(row, e)
    for e in np.flatnonzero((counts >= 1) & (counts <= 2)):
        for row in range(int(counts[e])):
            add(row, e)
    rng = np.random.default_rng(1000 + case.seed)
    for t in rng.permutation(T):
        if len(chosen) >= case.n_sample:
            break
        if int(t) not in chosen:
            chosen.append(int(t))
    return np.array(sorted(chosen))


def _inputs(case: Case):
    x = activations(case.T, BEAM, seed=case.seed)
    wr = router_weight(BEAM)
    bias = case.bias_scale * zipf_bias(BEAM.E) if case.bias_scale else None
    return x, wr, bias


def gpu_run(ex, case: Case, x, wr, bias, tokens):
    """One nvfp4moe_forward of the case with debug exports; returns the host copies of the
    routing, grouping, quantised input, the sampled tokens' outputs and their pairs'
    requantised intermediate ([tokens, topk, ...]), and the status word."""
    T, k = case.T, BEAM.topk
    ws = torch.empty(moe.forward_workspace_bytes(ex.cfg, T), dtype=torch.uint8, device="cuda")
    out, dbg = moe.forward(ex, x.cuda(), wr.cuda(), None if bias is None else bias.cuda(), ws=ws, debug=True,
                           debug_h=True)
    status = moe.status_read(ws)
    g = {n: dbg[n].cpu().numpy() for n in ("idx", "w", "counts", "offsets", "perm", "xq_codes", "xq_scales")}
    g["g_x"] = np.float32(dbg["g_x"].item())
    sel_t = torch.from_numpy(tokens).cuda()
    g["out"] = out[sel_t].float().cpu().numpy()
    g["acc"] = dbg["acc"][sel_t].cpu().numpy()
    # the BF16 output is the round-to-nearest-even of the FP32 sums, everywhere
    g["out_is_rounded_acc"] = bool(torch.equal(out, dbg["acc"].to(torch.bfloat16)))
    pos = np.empty(T * k, dtype=np.int64)
    pos[g["perm"]] = np.arange(T * k)
    pairs = (tokens[:, None] * k + np.arange(k)[None, :]).reshape(-1)
    sel = torch.from_numpy(pos[pairs]).cuda()
    hq_c = dbg["hq_codes"][sel].cpu().numpy().reshape(len(tokens), k, -1)
    hq_s = dbg["hq_scales"][sel].cpu().numpy().reshape(len(tokens), k, -1)
    g["h_f32"] = dbg["h_f32"][sel].cpu().numpy().reshape(len(tokens), k, -1)
    del out, dbg, ws
    torch.cuda.empty_cache()
    return g, hq_c, hq_s, status


@pytest.fixture(scope="module")
def runs():
    """GPU forward of every case (debug exports of the routing, grouping, quantised input and
    the requantised intermediate of the sampled pairs), then one oracle pass over the experts."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    return collect(gpu_experts(BEAM))


def collect(ex, cases=CASES):
    g_h = intermediate_scales(BEAM)
    cfg = cfg_ns(BEAM)
    res = {}
    jobs = {}          # expert -> rows [(case, token, slot, xhat, gpu hq codes, gpu hq scales)]
    for case in cases:
        x, wr, bias = _inputs(case)
        xn = x.float().numpy()
        bn = None if bias is None else bias.numpy().astype(np.float64)
        r = oracle.route(xn.astype(np.float64), wr.numpy().astype(np.float64), cfg, bn)
        tokens = pick_tokens(case, r)
        g, hq_c, hq_s, status = gpu_run(ex, case, x, wr, bias, tokens)
        xc, xs, gx = oracle.quantize(xn)
        rec = {"case": case, "x": xn, "wr": wr.numpy(), "bias": bn, "route": r, "tokens": tokens,
               "status": status, "gpu": g, "xq": (xc, xs, gx), "pairs": {}}
        same_tok = (g["idx"][tokens] == r.idx[tokens]).all(axis=1)
        xhat = oracle.dequantize(xc[tokens], xs[tokens], gx)
        for i, t in enumerate(tokens):
            if not same_tok[i]:
                continue
            for j in range(BEAM.topk):
                e = int(r.idx[t, j])
                jobs.setdefault(e, []).append((case.name, int(t), j, xhat[i], hq_c[i, j], hq_s[i, j]))
                rec["pairs"][(int(t), j)] = {"h_gpu": g["h_f32"][i, j]}
        res[case.name] = rec
    packed = {e: (np.stack([v[3] for v in rows]), float(g_h[e]), np.stack([v[4] for v in rows]),
                  np.stack([v[5] for v in rows])) for e, rows in jobs.items()}
    out = oracle_expert_pass(BEAM, packed)
    for e, rows in jobs.items():
        y, y_g, h, hc, hs, dh = out[e]
        for n, (name, t, j, _, gc, gs) in enumerate(rows):
            res[name]["pairs"][(t, j)].update({"e": e, "y": y[n], "y_gpu_hq": y_g[n], "h": h[n], "hq_codes": hc[n],
                                               "hq_scales": hs[n], "gpu_codes": gc, "gpu_scales": gs, "dh": dh[n]})
    return res


@pytest.mark.parametrize("name", [c.name for c in CASES])
def test_beam_layer(runs, name):
    rec = runs[name]
    case, r, g, tokens = rec["case"], rec["route"], rec["gpu"], rec["tokens"]
    assert rec["status"] == moe.OK
    x64 = rec["x"].astype(np.float64)
    clean, n_flag = check_routing(g["idx"], g["w"], r, x64, rec["wr"].astype(np.float64), rec["bias"], BEAM)
    # the layer input, quantised: bit-exact
    xc, xs, gx = rec["xq"]
    assert g["g_x"] == gx
    np.testing.assert_array_equal(g["xq_codes"], xc)
    np.testing.assert_array_equal(g["xq_scales"], xs)
    # the grouping of the GPU's routing (and so of the oracle's where they agree)
    check_grouping({k: torch.from_numpy(g[k]) for k in ("counts", "offsets", "perm")}, g["idx"], BEAM.E)
    # the sampled pairs reach the tiles they were picked for
    counts = g["counts"]
    assert counts.sum() == case.T * BEAM.topk
    # requantised intermediate: equal except at near-ties of the FP32 rounding
    g_h = intermediate_scales(BEAM)
    # the FP32 SwiGLU product of every sampled pair within the derived bound of the epilogue
    worst = 0.0
    for (t, j), p in rec["pairs"].items():
        err = np.abs(p["h_gpu"].astype(np.float64) - p["h"])
        ratio = float(np.max(err / p["dh"]))
        worst = max(worst, ratio)
        assert ratio <= 1.0, f"{name}: pair ({t},{j}) h off by {ratio:.3g} of its bound"
    n_el = n_diff = 0
    for (t, j), p in rec["pairs"].items():
        block_tie, elem_tie = requant_near_tie(p["h"], float(g_h[p["e"]]), p["dh"])
        sb = p["gpu_scales"] != p["hq_scales"]
        assert not (sb & ~block_tie).any(), f"{name}: pair ({t},{j}) block scale differs away from a near-tie"
        gc = oracle.formats.unpack_codes(p["gpu_codes"][None])[0]
        oc = oracle.formats.unpack_codes(p["hq_codes"][None])[0]
        diff = gc != oc
        assert not (diff & ~(elem_tie | np.repeat(sb, 16))).any(), \
            f"{name}: pair ({t},{j}) code differs away from a near-tie"
        n_el += diff.size
        n_diff += int(diff.sum())
    assert n_diff <= max(4, 1e-3 * n_el), f"{name}: {n_diff} of {n_el} intermediate codes differ"
    # outputs of the sampled tokens routed as the oracle routes them
    same = np.array([(g["idx"][t] == r.idx[t]).all() for t in tokens])
    assert same.mean() > 0.9
    ref_ops = np.zeros((int(same.sum()), BEAM.H))
    ref_ind = np.zeros_like(ref_ops)
    for i, t in enumerate(tokens[same]):
        for j in range(BEAM.topk):
            p = rec["pairs"][(int(t), j)]
            ref_ops[i] += r.w[t, j] * p["y_gpu_hq"]
            ref_ind[i] += r.w[t, j] * p["y"]
    # the FP32 sums within the layer tolerance; the BF16 output their rounding
    assert g["out_is_rounded_acc"]
    got = g["acc"][same]
    err, fro = check_output(got, ref_ops)
    err_ind = float(np.abs(got - ref_ind).max())
    fro_ind = float(np.linalg.norm(got - ref_ind) / np.linalg.norm(ref_ind))
    print(f"{name}: T={case.T}, {len(tokens)} sampled tokens ({int(same.sum())} routed as the oracle), "
          f"{n_flag} near-tie tokens, h error at most {worst:.3g} of its bound, "
          f"{n_diff}/{n_el} intermediate codes at near-ties; max |out| "
          f"{np.abs(ref_ops).max():.3f}; same operands: max-abs {err:.3g}, rel-Frobenius {fro:.3g}; "
          f"independent oracle: max-abs {err_ind:.3g}, rel-Frobenius {fro_ind:.3g}")


def test_samples_reach_later_and_partial_tiles(runs):
    """The sampled pairs of the large cases sit in second-or-later 128-row tiles and in
    partial last tiles of their experts' segments, and (under the strong bias) in experts
    holding one or two rows while most experts hold none."""
    for name in ("prefill_T4096", "skewed_T16384", "strong_skew_T2048", "T32768"):
        rec = runs[name]
        g = rec["gpu"]
        counts, offsets, perm = g["counts"], g["offsets"], g["perm"]
        pos = np.empty(len(perm), dtype=np.int64)
        pos[perm] = np.arange(len(perm))
        later = partial = tiny = 0
        for (t, j) in rec["pairs"]:
            e = int(g["idx"][t, j])
            row = pos[t * BEAM.topk + j] - offsets[e]
            later += row >= 128
            partial += row >= (counts[e] // 128) * 128
            tiny += counts[e] <= 2
        assert later >= 16 and partial >= 8, (name, later, partial)
        if name == "strong_skew_T2048":
            assert (counts == 0).sum() > 100 and tiny >= 10, (name, tiny)
