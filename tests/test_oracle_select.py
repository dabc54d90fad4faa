"""Pins of the oracle's budget and selection steps (no GPU): budget invariants,
brute force over all subsets on small heads, ties, signed zeros, segments."""
import itertools
import math

import numpy as np
import pytest

import synth
from oracle import veda_oracle as O


def _counts(k):
    vals, cnt = np.unique(k, return_counts=True)
    return dict(zip(vals.tolist(), cnt.tolist()))


@pytest.mark.parametrize("nT,rho,expect", [
    (496, (1, 10), {49: 199, 50: 297}),     # 16:9 clip: 24,601 blocks per head
    (64, (1, 10), {6: 39, 7: 25}),          # small workload: 409 blocks per head
    (4, (1, 2), {2: 4}),                    # tiny workload: 2 per row
    (496, (1, 20), {24: 100, 25: 396}),
    (992, (1, 10), {99: 794, 100: 198}),
])
def test_budget_counts(nT, rho, expect):
    k = O.budgets(nT, np.zeros(nT, int), [rho])[:, 0]
    assert _counts(k) == expect
    x = nT * rho[0] / rho[1]
    assert k.sum() == math.floor(nT * nT * rho[0] / rho[1])
    assert set(k.tolist()) <= {math.floor(x), math.ceil(x)}


def test_budget_diagonal_floor_and_clamp():
    seg = np.array([0] * 6 + [1] * 2)
    k = O.budgets(8, seg, [(1, 20), (1, 1)])
    assert (k[:6, 0] == 1).all()            # x = 0.3 would give 0: raised to 1 for the diagonal
    assert (k[6:, 0] == np.array([math.floor(7 * 0.3) - math.floor(6 * 0.3),
                                  math.floor(8 * 0.3) - math.floor(7 * 0.3)])).all()
    assert (k[:, 1] == 2).all()             # 100% of a 2-tile segment


def _brute_row(S_row, r, segment, k_row):
    """All subsets: per segment, maximise the score sum, then minimise the index sum."""
    chosen = []
    for s, kk in enumerate(k_row):
        cand = [j for j in range(len(segment)) if segment[j] == s]
        forced = [r] if segment[r] == s and kk > 0 else []
        pool = [j for j in cand if j not in forced]
        need = kk - len(forced)
        best = max(itertools.combinations(pool, need),
                   key=lambda c: (sum(0.0 + S_row[j] for j in c), -sum(c)))
        chosen.extend(forced + list(best))
    return sorted(chosen)


@pytest.mark.parametrize("seed", range(6))
def test_select_matches_brute_force(seed):
    rng = np.random.default_rng(seed)
    nT = 8
    S = rng.standard_normal((nT, nT))
    if seed % 2:
        S = np.round(S * 2) / 2                 # many exact ties
    seg = np.array([0] * 6 + [1] * 2) if seed >= 3 else np.zeros(nT, int)
    rho = [(3, 8), (1, 2)] if seed >= 3 else [(3, 8)]
    k = O.budgets(nT, seg, rho)
    for r in range(nT):
        got = O.select_row(S[r], r, seg, k[r]).tolist()
        assert got == _brute_row(S[r], r, seg, k[r])
        assert r in got and len(got) == k[r].sum()


def test_signed_zero_ties_and_nan():
    S_row = np.array([0.0, -0.0, 0.0, -1.0, -0.0])
    got = O.select_row(S_row, 4, np.zeros(5, int), np.array([3]))
    assert got.tolist() == [0, 1, 4]            # -0 == +0, so index order decides
    with pytest.raises(ValueError):
        O.select_row(np.array([0.0, np.nan]), 0, np.zeros(2, int), np.array([2]))


def test_full_density_takes_everything_and_split():
    nT = 5
    S = np.random.default_rng(9).standard_normal((1, 1, nT, nT))
    nv = np.array([[128, 128, 7, 128, 1]])
    lists = O.select(S, nv, np.zeros((1, nT), int), [nT], [(1, 1)])
    for r in range(nT):
        assert lists.full[0][0][r].tolist() == [0, 1, 3]
        assert lists.partial[0][0][r].tolist() == [2, 4]


def test_rows_past_head_count_are_empty():
    S = np.zeros((1, 2, 4, 4))
    nv = np.array([[128] * 4, [128, 128, 0, 0]])
    seg = np.zeros((2, 4), int)
    lists = O.select(S, nv, seg, [4, 2], [(1, 2)])
    assert [len(lists.full[0][1][r]) for r in range(4)] == [1, 1, 0, 0]


def test_every_row_keeps_diagonal_and_budget_small_workload():
    w = synth.SMALL
    rng = np.random.default_rng(2)
    nT = w.nT
    S = rng.standard_normal((1, 1, nT, nT))
    nv = np.full((1, nT), 128)
    lists = O.select(S, nv, np.zeros((1, nT), int), [nT], w.rho)
    tot = 0
    for r in range(nT):
        sel = np.concatenate([lists.full[0][0][r], lists.partial[0][0][r]])
        assert r in sel and len(set(sel.tolist())) == len(sel)
        assert (np.diff(lists.full[0][0][r]) > 0).all()
        tot += len(sel)
    assert tot == 409
