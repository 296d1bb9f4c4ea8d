"""Pins for the oracle router (CPU only): brute force over every admissible
selection on the tiny layer, the plain top-k special case, a hand-worked example
and the weight invariants."""
import itertools
import types

import numpy as np
import torch

import oracle
from workloads import TINY, activations, router_weight


def _cfg(E, G, KG, K, rho=2.5):
    return types.SimpleNamespace(E=E, n_groups=G, topk_groups=KG, topk=K, routed_scale=rho)


def _brute_force(s, E, G, KG, K):
    """Best (group set, expert subset) over every admissible choice, lexicographically:
    first the summed group score (each group's two best scores), then the summed
    expert score; all choices are enumerated."""
    gs = E // G
    gscore = np.array([np.sort(s[g * gs:(g + 1) * gs])[-2:].sum() for g in range(G)])
    best = None
    for gset in itertools.combinations(range(G), KG):
        gsum = gscore[list(gset)].sum()
        if best is not None and gsum < best[0]:
            continue
        cand = np.array([e for g in gset for e in range(g * gs, (g + 1) * gs)])
        combos = np.array(list(itertools.combinations(range(len(cand)), K)))
        sums = s[cand[combos]].sum(axis=1)
        i = int(np.argmax(sums))
        key = (gsum, sums[i])
        if best is None or key > best[:2]:
            best = (gsum, sums[i], set(cand[combos[i]].tolist()))
    return best[2]


def test_router_matches_brute_force_on_tiny_layer():
    cfg = _cfg(TINY.E, TINY.n_groups, TINY.topk_groups, TINY.topk)
    x = activations(12, TINY).float().numpy()
    wr = router_weight(TINY).numpy()
    r = oracle.route(x, wr, cfg)
    for t in range(x.shape[0]):
        assert set(r.idx[t].tolist()) == _brute_force(r.scores[t], TINY.E, 8, 4, 8)


def test_single_group_reduces_to_plain_topk():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((50, 64))
    wr = rng.standard_normal((40, 64)) / 8
    r = oracle.route(x, wr, _cfg(40, 1, 1, 6))
    s = 1 / (1 + np.exp(-(x @ wr.T)))
    want = np.argsort(-s, axis=1, kind="stable")[:, :6]
    np.testing.assert_array_equal(r.idx, want)


def test_hand_worked_example():
    # 8 experts in 4 groups of 2, keep 2 groups, pick 3 experts; logits chosen so the
    # sigmoid order is the logit order.  Group sums (of both members):
    #   g0 = {e0: 3.0, e1: -3.0}  -> s ~ 0.953 + 0.047 = 1.000
    #   g1 = {e2: 1.0, e3:  0.9}  -> s ~ 0.731 + 0.711 = 1.442
    #   g2 = {e4: 2.0, e5: -2.0}  -> s ~ 0.881 + 0.119 = 1.000 (tie with g0 -> g0 wins)
    #   g3 = {e6: 0.5, e7:  0.4}  -> s ~ 0.622 + 0.599 = 1.221
    # Kept groups: g1, g3.  Best 3 of {e2, e3, e6, e7}: e2, e3, e6.
    logits = np.array([[3.0, -3.0, 1.0, 0.9, 2.0, -2.0, 0.5, 0.4]])
    # x = ones and W = diag(l) give logit_e = l_e
    r = oracle.route(np.ones((1, 8)), np.diag(logits[0]), _cfg(8, 4, 2, 3))
    assert list(r.groups[0]) == [1, 3]
    assert list(r.idx[0]) == [2, 3, 6]
    s = 1 / (1 + np.exp(-np.array([1.0, 0.9, 0.5])))
    np.testing.assert_allclose(r.w[0], 2.5 * s / s.sum(), rtol=1e-15)


def test_weights_sum_to_routed_scale_and_follow_scores():
    cfg = _cfg(TINY.E, TINY.n_groups, TINY.topk_groups, TINY.topk)
    x = activations(64, TINY).float().numpy()
    r = oracle.route(x, router_weight(TINY).numpy(), cfg)
    np.testing.assert_allclose(r.w.sum(axis=1), 2.5, rtol=1e-14)
    sel = np.take_along_axis(r.scores, r.idx, axis=1)
    np.testing.assert_allclose(r.w / r.w[:, :1], sel / sel[:, :1], rtol=1e-13)
    assert np.all(np.diff(sel, axis=1) <= 0)                        # score descending
    assert np.all(r.expert_margin >= 0) and np.all(r.group_margin >= 0)
    # selected experts lie in the kept groups
    assert np.all(np.isin(r.idx // (TINY.E // TINY.n_groups), r.groups).all(axis=1))


def test_single_expert_weight_is_routed_scale():
    rng = np.random.default_rng(3)
    r = oracle.route(rng.standard_normal((5, 16)), rng.standard_normal((8, 16)), _cfg(8, 2, 1, 1))
    np.testing.assert_allclose(r.w, 2.5)


def test_bias_shifts_selection():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((20, 32))
    wr = rng.standard_normal((32, 32)) / 6
    bias = np.zeros(32)
    bias[17] = 50.0
    r = oracle.route(x, wr, _cfg(32, 8, 4, 8), bias=bias)
    assert np.all(r.idx[:, 0] == 17)


def test_bias_is_a_logit_offset():
    """The skewed workload's per-expert bias is added to the logits before the sigmoid: it
    routes exactly like one more input column of ones whose router weights are the bias.
    Inputs are integers scaled by powers of two, so both forms give the same FP64 logits."""
    rng = np.random.default_rng(5)
    x = rng.integers(-8, 9, size=(40, 32)) / 8.0
    wr = rng.integers(-8, 9, size=(32, 32)) / 64.0
    bias = rng.integers(-16, 17, size=32) / 8.0
    cfg = _cfg(32, 8, 4, 8)
    r = oracle.route(x, wr, cfg, bias=bias)
    r1 = oracle.route(np.hstack([x, np.ones((40, 1))]), np.hstack([wr, bias[:, None]]), cfg)
    np.testing.assert_array_equal(r.idx, r1.idx)
    np.testing.assert_array_equal(r.w, r1.w)


def test_bias_alone_gives_sigmoid_of_bias():
    """With x = 0 the scores are the sigmoid of the bias, and the weights its normalised
    selection scaled by 2.5 (closed form)."""
    bias = np.linspace(-2.0, 2.0, 16)
    r = oracle.route(np.zeros((1, 8)), np.zeros((16, 8)), _cfg(16, 1, 1, 4), bias=bias)
    sig = 1.0 / (1.0 + np.exp(-bias))
    assert list(r.idx[0]) == [15, 14, 13, 12]
    np.testing.assert_allclose(r.w[0], 2.5 * sig[[15, 14, 13, 12]] / sig[12:].sum(), rtol=1e-15)


def test_ties_go_to_lower_index():
    x = np.ones((1, 4))
    wr = np.zeros((8, 4))                 # every score equal
    r = oracle.route(x, wr, _cfg(8, 4, 2, 3))
    assert list(r.groups[0]) == [0, 1] and list(r.idx[0]) == [0, 1, 2]


def test_decision_margins_by_sorting():
    """The margins the parity protocol uses to tell FP32 near-ties from mismatches, rebuilt with
    Python sorts from sigmoid scores the test computes itself: the last kept group's score minus
    the best dropped group's, the last selected expert's score minus the best unselected
    admissible one's, and the smallest gap between consecutive selected scores."""
    cfg = _cfg(TINY.E, TINY.n_groups, TINY.topk_groups, TINY.topk)
    x = activations(16, TINY).float().numpy().astype(np.float64)
    wr = router_weight(TINY).numpy().astype(np.float64)
    r = oracle.route(x, wr, cfg)
    s = 1 / (1 + np.exp(-(x @ wr.T)))
    gs = TINY.E // TINY.n_groups
    for t in range(x.shape[0]):
        gsc = [sum(sorted(s[t, g * gs:(g + 1) * gs].tolist(), reverse=True)[:2]) for g in range(TINY.n_groups)]
        gord = sorted(range(TINY.n_groups), key=lambda g: (-gsc[g], g))
        np.testing.assert_allclose(r.group_margin[t], gsc[gord[3]] - gsc[gord[4]], rtol=1e-12, atol=0)
        cand = sorted((e for g in gord[:4] for e in range(g * gs, (g + 1) * gs)), key=lambda e: (-s[t, e], e))
        np.testing.assert_allclose(r.expert_margin[t], s[t, cand[7]] - s[t, cand[8]], rtol=1e-12, atol=0)
        sel = [s[t, e] for e in cand[:8]]
        np.testing.assert_allclose(r.order_margin[t], min(a - b for a, b in zip(sel, sel[1:])), rtol=1e-12, atol=0)
