"""Pins of the oracle's attention step and of the whole path (no GPU).

* at 100% density the tiled block-sparse path equals dense softmax attention in
  raster order (an untiled routine);
* an explicit token-level mask in raster order reproduces the tiled result for
  any block lists;
* a one-block row is the textbook softmax over that tile's valid keys;
* identical keys give the plain mean of the values.
"""
import numpy as np
import pytest

import synth
from oracle import veda_oracle as O

SCALE = 1.0 / np.sqrt(128)


def _inputs(B, N, H, seed):
    rng = np.random.default_rng(seed)
    q, k, v = rng.standard_normal((3, B, N, H, 128))
    W = 0.02 * rng.standard_normal((2, H, 128, 384))
    return q, k, v, W[0], W[1]


@pytest.mark.parametrize("grid,shapes,tail", [
    ((4, 8, 16), [(1, 8, 16), (1, 8, 16)], 0),
    ((3, 9, 20), [(1, 8, 16), (2, 8, 8)], 0),
    ((2, 8, 12), [(4, 4, 8)], 77),
])
def test_full_density_equals_dense_raster(grid, shapes, tail):
    H = len(shapes)
    N = grid[0] * grid[1] * grid[2] + tail
    q, k, v, Wq, Wk = _inputs(1, N, H, 11)
    rho = [(1, 1), (1, 1)] if tail else [(1, 1)]
    out = O.run_path(q, k, v, Wq, Wk, grid, shapes, tail, rho, SCALE)
    od, lsed = O.dense_attention_raster(q, k, v, SCALE)
    assert np.allclose(out["o"], od, rtol=1e-12, atol=1e-12)
    for h in range(H):
        sl = out["slots"][h]
        ok = sl >= 0
        assert np.allclose(out["lse"][0, h, ok], lsed[0, sl[ok], h], rtol=1e-12, atol=1e-12)


def _token_mask_attention(q, k, v, slots, lists, N, scale):
    """Raster-order attention with an explicit token x token mask built from the lists."""
    B, _, H, D = q.shape
    o = np.zeros((B, N, H, D))
    for b in range(B):
        for h in range(H):
            tile_of = np.full(N, -1)
            for s in np.flatnonzero(slots[h] >= 0):
                tile_of[slots[h, s]] = s // 128
            M = np.zeros((N, N), bool)
            for i in range(N):
                r = tile_of[i]
                keys = np.concatenate([lists.full[b][h][r], lists.partial[b][h][r]])
                M[i] = np.isin(tile_of, keys)
            s_ = scale * q[b, :, h] @ k[b, :, h].T
            s_ = np.where(M, s_, -np.inf)
            p = np.exp(s_ - s_.max(axis=1, keepdims=True))
            o[b, :, h] = (p / p.sum(axis=1, keepdims=True)) @ v[b, :, h]
    return o


@pytest.mark.parametrize("grid,shape,tail,rho", [
    ((4, 8, 16), (1, 8, 16), 0, [(1, 2)]),
    ((3, 9, 20), (2, 8, 8), 0, [(1, 3)]),
    ((2, 8, 12), (4, 4, 8), 150, [(1, 2), (1, 2)]),
])
def test_sparse_path_equals_token_mask(grid, shape, tail, rho):
    N = grid[0] * grid[1] * grid[2] + tail
    q, k, v, Wq, Wk = _inputs(1, N, 2, 12)
    order = [None, np.random.default_rng(4).permutation(O.tile_map(grid, shape).n_valid.size)]
    out = O.run_path(q, k, v, Wq, Wk, grid, [shape, shape], tail, rho, SCALE, tile_orders=order)
    ref = _token_mask_attention(q, k, v, out["slots"], out["lists"], N, SCALE)
    assert np.allclose(out["o"], ref, rtol=1e-12, atol=1e-12)
    # sparse really is sparse: it differs from dense
    od, _ = O.dense_attention_raster(q, k, v, SCALE)
    assert np.abs(out["o"] - od).max() > 1e-3


def test_one_block_row_is_softmax_over_its_tile():
    rng = np.random.default_rng(3)
    qt = rng.standard_normal((256, 128))
    kt = rng.standard_normal((256, 128))
    vt = rng.standard_normal((256, 128))
    nv = np.array([128, 50])
    o, lse = O.attention_row_tile(qt[:128], kt, vt, np.array([1]), nv, 0.3)
    s = 0.3 * qt[:128] @ kt[128:178].T
    e = np.exp(s)
    assert np.allclose(o, (e / e.sum(1, keepdims=True)) @ vt[128:178], rtol=1e-12, atol=1e-12)
    assert np.allclose(lse, np.log(e.sum(1)), rtol=1e-12)


def test_identical_keys_average_values():
    rng = np.random.default_rng(4)
    qt = rng.standard_normal((128, 128))
    kt = np.tile(rng.standard_normal(128), (384, 1))
    vt = rng.standard_normal((384, 128))
    nv = np.array([128, 128, 3])
    o, _ = O.attention_row_tile(qt, kt, vt, np.array([0, 2]), nv, SCALE)
    ref = np.concatenate([vt[0:128], vt[256:259]]).mean(0)
    assert np.allclose(o, ref[None, :], rtol=1e-12, atol=1e-12)


def test_empty_row_gives_zero_and_minus_inf():
    o, lse = O.attention_row_tile(np.ones((128, 128)), np.ones((128, 128)), np.ones((128, 128)),
                                  np.zeros(0, int), np.array([128]), SCALE)
    assert (o == 0).all() and np.isneginf(lse).all()


def test_tiny_workload_path_runs_and_is_finite():
    w = synth.TINY
    x = synth.make_inputs(w)
    f = lambda t: t.double().numpy()
    out = O.run_path(f(x.q), f(x.k), f(x.v), f(x.wq), f(x.wk), w.grid, w.head_shapes, w.n_tail,
                     w.rho, SCALE)
    assert np.isfinite(out["o"]).all()
    counts = [[len(out["lists"].full[0][h][r]) for r in range(4)] for h in range(2)]
    assert counts == [[2] * 4, [2] * 4]
