"""The claim order of the one-launch decode GEMMs, modelled on the CPU.

At decode the gate/up and down grouped GEMMs run as one persistent launch: every CTA claims
work items in one global order, and a down item's producer waits (bounded) until all gate/up
items of its 128-row tile have stored their part of h.  A claimed gate/up item never waits,
so the launch cannot deadlock when

  (a) the order is a permutation of all gate/up and down items, and
  (b) every gate/up item of a row tile comes before every down item of that tile.

The order (csrc/gemm.cu, decode_fused): the gate/up items keep their own order (expert-major,
then 256-column tile, then row tile); expert e's down items, in the same order, form one
block claimed after the first min(G(e + 1) + lag, NG) gate/up items, G(e) counting the
gate/up items of the experts before e and NG all of them.  This test restates that index
arithmetic (the binary searches over the experts' row-tile prefix included) and checks (a),
(b) and the lag between an expert's last gate/up item and its first down item, on random
row-tile layouts with empty experts, on one rank's share of the experts (a prefix that
starts at a later row tile) and on the Beam decode layout.
"""
import numpy as np
import pytest


def decode_work(prefix, w, E, ntn):
    """Item w of one GEMM's order -> (expert, column tile, global row tile)."""
    lo, hi = 0, E
    while hi - lo > 1:
        mid = (lo + hi) >> 1
        if prefix[mid] * ntn <= w:
            lo = mid
        else:
            hi = mid
    p_lo, mt_e = prefix[lo], prefix[lo + 1] - prefix[lo]
    local = w - p_lo * ntn
    nt = local // mt_e
    return lo, nt, p_lo + (local - nt * mt_e)


def decode_fused(prefix, E, ntn_g, ntn_d, lag, w):
    """Claim w of the one-launch order -> (is gate/up, expert, column tile, global row tile)."""
    base = prefix[0]
    NG = (prefix[E] - base) * ntn_g

    def start(e):
        g1 = (prefix[e + 1] - base) * ntn_g + lag
        return min(g1, NG) + (prefix[e] - base) * ntn_d

    lo, hi = -1, E
    while hi - lo > 1:
        mid = (lo + hi) >> 1
        if start(mid) <= w:
            lo = mid
        else:
            hi = mid
    g = w
    if lo >= 0:
        s0 = start(lo)
        p_lo, mt_e = prefix[lo], prefix[lo + 1] - prefix[lo]
        if w < s0 + mt_e * ntn_d:
            return (False,) + decode_work(prefix, (p_lo - base) * ntn_d + (w - s0) + base * ntn_d, E, ntn_d)
        g = w - (p_lo + mt_e - base) * ntn_d
    return (True,) + decode_work(prefix, g + base * ntn_g, E, ntn_g)


def _check(tiles, ntn_g, ntn_d, lag, base=0):
    E = len(tiles)
    prefix = [base] + list(base + np.cumsum(tiles))
    m_total = prefix[E] - base
    NG, ND = m_total * ntn_g, m_total * ntn_d
    order = [decode_fused(prefix, E, ntn_g, ntn_d, lag, w) for w in range(NG + ND)]
    # (a) a permutation of every item
    want = {(True, e, nt, prefix[e] + m) for e in range(E) for nt in range(ntn_g) for m in range(tiles[e])}
    want |= {(False, e, nt, prefix[e] + m) for e in range(E) for nt in range(ntn_d) for m in range(tiles[e])}
    assert len(order) == len(set(order)) and set(order) == want
    pos = {item: w for w, item in enumerate(order)}
    # gate/up items keep their own order
    gu = [item for item in order if item[0]]
    assert gu == [(True,) + decode_work(prefix, g + base * ntn_g, E, ntn_g) for g in range(NG)]
    for e in range(E):
        if tiles[e] == 0:
            continue
        rows = range(prefix[e], prefix[e + 1])
        last_gu = max(pos[(True, e, nt, m)] for nt in range(ntn_g) for m in rows)
        downs = [pos[(False, e, nt, m)] for nt in range(ntn_d) for m in rows]
        # (b) every gate/up item of the expert's row tiles before any of its down items
        assert last_gu < min(downs)
        # the down items form one contiguous block
        assert max(downs) - min(downs) == len(downs) - 1
        # gate/up items claimed between the expert's last gate/up item and its down block
        g_end = (prefix[e + 1] - base) * ntn_g
        between = sum(1 for w in range(last_gu + 1, min(downs)) if order[w][0])
        assert between == min(lag, NG - g_end)


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("lag", [0, 1, 7, 592])
def test_random_layouts_with_empty_experts(seed, lag):
    rng = np.random.default_rng(seed)
    E = int(rng.choice([1, 2, 8, 32]))
    tiles = rng.integers(0, 3, size=E)
    if tiles.sum() == 0:
        tiles[rng.integers(E)] = 1
    _check(list(tiles), ntn_g=int(rng.integers(1, 5)), ntn_d=int(rng.integers(1, 5)), lag=lag)


@pytest.mark.parametrize("lag", [0, 5, 592])
def test_one_ranks_share_of_the_experts(lag):
    """A local handle's launch sees the prefix from its first expert on: row tiles start at a
    later global number."""
    _check([1, 0, 2, 1, 0, 3], ntn_g=3, ntn_d=2, lag=lag, base=37)


def test_beam_decode_layout():
    """Beam at T = 16: 99 experts hit with one row tile each among 256, 20 column tiles of
    256 in both GEMMs (2 I / 256 and H / 256), lag 4 x 148 claims."""
    rng = np.random.default_rng(11)
    tiles = np.zeros(256, dtype=np.int64)
    tiles[rng.choice(256, size=99, replace=False)] = 1
    _check(list(tiles), ntn_g=20, ntn_d=20, lag=4 * 148)
