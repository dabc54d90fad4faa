"""Pins of the oracle tile-plan search (no GPU).

* at density 1/1 every shape keeps every block and its error is 0;
* the error of a shape equals the one computed on an independent route: a token x token
  mask in raster order built from the oracle mask's lists, applied to a textbook masked
  softmax (no tiled layout, no unpermute);
* the vote: hand-worked cases for "each head's best shape, the two most voted shapes kept,
  each head takes its better kept shape", with the stated tie rules.
"""
import numpy as np
import pytest

from oracle import veda_oracle as O

SCALE = 1.0 / np.sqrt(128)
CANDIDATES = [(1, 8, 16), (2, 8, 8), (4, 4, 8)]


def _inputs(grid, H, seed):
    N = grid[0] * grid[1] * grid[2]
    rng = np.random.default_rng(seed)
    q, k, v = rng.standard_normal((3, 1, N, H, 128))
    k += 0.7 * q                                   # attention far from uniform
    return q, k, v


def test_full_density_has_no_error():
    grid = (4, 8, 16)
    q, k, v = _inputs(grid, 2, 3)
    err = O.shape_errors(q, k, v, grid, 0, CANDIDATES, [(1, 1)], SCALE)
    assert np.all(err < 1e-20)


def test_error_matches_token_mask_route():
    grid = (4, 8, 16)
    q, k, v = _inputs(grid, 1, 4)
    rho = [(1, 4)]
    err = O.shape_errors(q, k, v, grid, 0, CANDIDATES, rho, SCALE)
    N = q.shape[1]
    od, _ = O.dense_attention_raster(q, k, v, SCALE)
    for ci, shape in enumerate(CANDIDATES):
        m = O.tile_map(grid, shape, 0)
        slots, nv, seg = O.stack_maps([m])
        qt, kt = O.permute(q, slots), O.permute(k, slots)
        heat = O.block_heat(qt, kt, nv, [len(m.n_valid)], SCALE)
        lists = O.select(heat, nv, seg, [len(m.n_valid)], rho)
        tile_of = np.full(N, -1)
        for s_ in np.flatnonzero(slots[0] >= 0):
            tile_of[slots[0, s_]] = s_ // 128
        M = np.zeros((N, N), bool)
        for i in range(N):
            r = tile_of[i]
            M[i] = np.isin(tile_of, np.concatenate([lists.full[0][0][r], lists.partial[0][0][r]]))
        s_ = np.where(M, SCALE * q[0, :, 0] @ k[0, :, 0].T, -np.inf)
        p = np.exp(s_ - s_.max(axis=1, keepdims=True))
        o = (p / p.sum(axis=1, keepdims=True)) @ v[0, :, 0]
        ref = ((o - od[0, :, 0]) ** 2).sum() / (od[0, :, 0] ** 2).sum()
        assert err[0, ci] == pytest.approx(ref, rel=1e-10)
        assert 0 < err[0, ci] < 1


def test_vote_hand_examples():
    # 5 heads, 3 candidates: best shapes 0, 2, 2, 1, 2 -> keep {2, 0} (votes 3, then 1 vs 1: the
    # earlier, 0); heads take their better kept shape
    err = np.array([[0.1, 0.2, 0.3],
                    [0.5, 0.4, 0.3],
                    [0.9, 0.8, 0.1],
                    [0.3, 0.1, 0.4],
                    [0.6, 0.6, 0.5]])
    kept, assign = O.tile_plan(err)
    assert kept == [0, 2]
    assert assign.tolist() == [0, 2, 2, 0, 2]
    # one shape wins every head: only it is kept
    kept, assign = O.tile_plan(np.array([[0.1, 0.2], [0.2, 0.3]]))
    assert kept == [0] and assign.tolist() == [0, 0]
    # equal errors: the earlier candidate
    kept, assign = O.tile_plan(np.array([[0.2, 0.2, 0.2]]), max_shapes=1)
    assert kept == [0] and assign.tolist() == [0]
