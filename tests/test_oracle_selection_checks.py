"""The oracle's top-K ranking and its top-K validity check against plain
per-row Python on inputs with many ties (scores rounded to 2 decimals)."""

import numpy as np
import pytest

from oracle import gsa_oracle as O


def _plain_valid(geo, g_row, chosen, window):
    ids = [int(b) for b in chosen if b >= 0]
    if len(ids) != geo.K_eff or len(set(ids)) != len(ids):
        return False
    if any(not (geo.B0 <= b < geo.NB) for b in ids):
        return False
    rest = [g_row[b] for b in range(geo.B0, geo.NB) if b not in ids]
    if not rest or not ids:
        return True
    return max(rest) - min(g_row[b] for b in ids) < window


@pytest.mark.parametrize("keep", ["specials", "reference"])
def test_ranking_and_validity_against_plain_python(keep):
    rng = np.random.default_rng(1)
    geo = O.Geometry(N=3, S=1, Hp=8, Wp=8, H=2, D=8, P=4, K=5, keep=keep)
    for it in range(60):
        g = np.round(rng.normal(size=(4, 2, geo.NB)), 2)
        own = O.top_k_blocks(geo, g)
        for r in range(4):
            for h in range(2):
                want = sorted(range(geo.B0, geo.NB), key=lambda b: (-g[r, h, b], b))[:geo.K_eff]
                assert [b for b in own[r, h] if b >= 0] == sorted(want)
        assert O.selection_valid_top_k(geo, g, own, 1e-12).all()
        other = own.copy()
        other[0, 0, rng.integers(geo.K_eff)] = rng.integers(geo.B0, geo.NB)  # maybe a duplicate
        other[1, 1, 0] = -1                                                 # one id short
        other[2, 0, 1] = other[2, 0, 0] + 1 if it % 2 else other[2, 0, 1]   # maybe a weaker block
        got = O.selection_valid_top_k(geo, g, other, 0.05)
        for r in range(4):
            for h in range(2):
                assert got[r, h] == _plain_valid(geo, g[r, h], other[r, h], 0.05)


@pytest.mark.parametrize("keep", ["specials", "reference"])
def test_gap_against_plain_sort(keep):
    # the K-th minus the (K+1)-th largest candidate score, inf when every
    # candidate is selected; the parity tests' tie window is read from it
    rng = np.random.default_rng(2)
    for K in (1, 5, 20, 32):
        geo = O.Geometry(N=3, S=1, Hp=8, Wp=8, H=2, D=8, P=4, K=K, keep=keep)
        g = np.round(rng.normal(size=(3, 2, geo.NB)), 2)
        gap = O.top_k_gap(geo, g)
        for r in range(3):
            for h in range(2):
                cand = sorted(g[r, h, geo.B0:], reverse=True)
                want = np.inf if geo.K_eff >= len(cand) else cand[geo.K_eff - 1] - cand[geo.K_eff]
                assert gap[r, h] == want


def _two_pass(geo, g_row, first):
    # the first pass keeps the `first` best (score, lower id) pairs and records
    # the worst of them; the second keeps the next K - first pairs strictly below
    # that pair in the same order; the selection is their union
    order = sorted(range(geo.B0, geo.NB), key=lambda b: (-g_row[b], b))
    top = order[:first]
    if len(top) < first:
        return sorted(top)
    bound = (-g_row[top[-1]], top[-1])
    rest = [b for b in order if (-g_row[b], b) > bound][:geo.K_eff - first]
    return sorted(top + rest)


@pytest.mark.parametrize("K", [65, 100, 128])
def test_two_ranking_passes_equal_the_top_k(K):
    # the reading behind gsa_forward's K > 64 path: ranking the first 64 and then
    # the next K - 64 strictly below the 64th pair is exactly the top-K, ties to
    # the lower id included
    rng = np.random.default_rng(3)
    for keep in ("specials", "reference"):
        geo = O.Geometry(N=4, S=1, Hp=20, Wp=20, H=1, D=8, P=4, K=K, keep=keep)
        g = np.round(rng.normal(size=(6, 1, geo.NB)), 1)  # many ties
        own = O.top_k_blocks(geo, g)
        for r in range(6):
            assert _two_pass(geo, g[r, 0], 64) == [b for b in own[r, 0] if b >= 0]
