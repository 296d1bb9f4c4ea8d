"""Group-limited sigmoid router, in FP64.  TEST INFRASTRUCTURE ONLY.

Follows "Reflection releases Beam ...", section "Mixture-of-Experts details":
the router scores every expert with a sigmoid, splits the experts into groups,
keeps the ``topk_groups`` groups whose two best scores sum highest, selects the
``topk`` best experts inside the kept groups, and the outputs are combined with
the normalised router weights times 2.5.  The pages keep the router unquantised
("NVFP4 quantization", section "Quantization scheme") and compute it in FP32
(section "Residual stream and numerical decisions" of the Beam summary); the
oracle computes it exactly (FP64) and reports decision margins so a test can
tell a genuine mismatch from an FP32 near-tie.

Readings where the pages are silent: groups are contiguous blocks of experts;
ties between equal scores go to the lower group / expert index; the selected
experts are listed by score descending (then index ascending); the weights are
normalised over the selected sigmoid scores and multiplied by the routed scale
afterwards; an optional per-expert logit bias is added before the sigmoid (the
pages give none; it exists only to build a skewed synthetic workload).
"""
from __future__ import annotations

import dataclasses

import numpy as np


@dataclasses.dataclass
class RouteResult:
    idx: np.ndarray          # int64 [T, k]   selected experts, score descending
    w: np.ndarray            # float64 [T, k] routed_scale * s / sum(s_selected)
    logits: np.ndarray       # float64 [T, E]
    scores: np.ndarray       # float64 [T, E] sigmoid
    group_scores: np.ndarray  # float64 [T, G] sum of the two best scores per group
    groups: np.ndarray       # int64 [T, topk_groups] kept groups, best first
    group_margin: np.ndarray  # float64 [T] score of last kept group minus best dropped (inf if none)
    expert_margin: np.ndarray  # float64 [T] last selected minus best unselected admissible (inf if none)
    order_margin: np.ndarray   # float64 [T] smallest gap between consecutive selected scores


def _sigmoid(l):
    return 1.0 / (1.0 + np.exp(-l))


def route(x, w_router, cfg, bias=None) -> RouteResult:
    """Route T tokens.

    x: [T, H] (BF16 values, any float dtype), w_router: [E, H], bias: [E] or None.
    cfg: object with E, n_groups, topk_groups, topk, routed_scale.
    """
    x = np.asarray(x, dtype=np.float64)
    wr = np.asarray(w_router, dtype=np.float64)
    T = x.shape[0]
    E, G, KG, K = cfg.E, cfg.n_groups, cfg.topk_groups, cfg.topk
    gs = E // G
    logits = x @ wr.T
    if bias is not None:
        logits = logits + np.asarray(bias, dtype=np.float64)[None, :]
    s = _sigmoid(logits)

    grp = s.reshape(T, G, gs)
    top2 = -np.sort(-grp, axis=2)[:, :, : min(2, gs)]
    gscore = top2.sum(axis=2)

    gidx = np.arange(G)
    idx = np.zeros((T, K), dtype=np.int64)
    w = np.zeros((T, K), dtype=np.float64)
    groups = np.zeros((T, KG), dtype=np.int64)
    gmargin = np.full(T, np.inf)
    emargin = np.full(T, np.inf)
    omargin = np.full(T, np.inf)
    eidx = np.arange(E)
    for t in range(T):
        gorder = np.lexsort((gidx, -gscore[t]))          # score desc, then index asc
        kept = np.sort(gorder[:KG])
        groups[t] = gorder[:KG]
        if G > KG:
            gmargin[t] = gscore[t, gorder[KG - 1]] - gscore[t, gorder[KG]]
        admissible = (eidx // gs)[None, :] == kept[:, None]
        cand = eidx[admissible.any(axis=0)]
        corder = cand[np.lexsort((cand, -s[t, cand]))]    # score desc, then index asc
        sel = corder[:K]
        if len(corder) > K:
            emargin[t] = s[t, corder[K - 1]] - s[t, corder[K]]
        idx[t] = sel
        ss = s[t, sel]
        if K > 1:
            omargin[t] = np.min(ss[:-1] - ss[1:])
        w[t] = cfg.routed_scale * ss / ss.sum()
    return RouteResult(idx, w, logits, s, gscore, groups, gmargin, emargin, omargin)
