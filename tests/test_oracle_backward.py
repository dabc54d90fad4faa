"""Pins of the oracle's attention backward and transposed lists (no GPU).

* at 100% density the tiled backward equals torch autograd of textbook dense attention in
  raster order (a library routine on an independent route: no tiling, no LSE);
* on a block-sparse case, central finite differences of the loss sum(O * G), with O the
  oracle's own block-sparse forward, match the backward's entries for Q, K and V;
* transposed lists: j is listed for query tile i exactly when i is listed for key tile j,
  ascending; a planted mistake (a dropped entry) is caught.
"""
import numpy as np
import pytest
import torch

from oracle import veda_oracle as O

SCALE = 1.0 / np.sqrt(128)


def _case(grid, shapes, tail, seed, rho):
    H = len(shapes)
    N = grid[0] * grid[1] * grid[2] + tail
    rng = np.random.default_rng(seed)
    q, k, v, g = rng.standard_normal((4, 1, N, H, 128))
    W = 0.02 * rng.standard_normal((2, H, 128, 384))
    out = O.run_path(q, k, v, W[0], W[1], grid, shapes, tail, rho, SCALE)
    return q, k, v, g, out


@pytest.mark.parametrize("grid,shapes,tail", [
    ((2, 8, 20), [(1, 8, 16)], 0),
    ((2, 8, 12), [(4, 4, 8), (1, 8, 16)], 77),
])
def test_full_density_equals_autograd_of_dense_attention(grid, shapes, tail):
    rho = [(1, 1), (1, 1)] if tail else [(1, 1)]
    q, k, v, g, out = _case(grid, shapes, tail, 21, rho)
    slots = out["slots"]
    dot = O.permute(g, slots)
    dq, dk, dv = O.attention_backward(out["q_tiled"], out["k_tiled"], out["v_tiled"], out["n_valid"],
                                      out["lists"], SCALE, np.nan_to_num(out["o_tiled"]), out["lse"], dot)
    N, H = q.shape[1], q.shape[2]
    for h in range(H):
        Q, K, V = (torch.tensor(x[0, :, h], requires_grad=True) for x in (q, k, v))
        Od = torch.softmax(SCALE * Q @ K.T, dim=1) @ V
        (Od * torch.from_numpy(g[0, :, h])).sum().backward()
        for grad, ref in ((dq, Q.grad), (dk, K.grad), (dv, V.grad)):
            raster = O.unpermute(grad[:, h:h + 1], slots[h:h + 1], N)[0, :, 0]
            assert np.allclose(raster, ref.numpy(), rtol=1e-10, atol=1e-12)


def test_sparse_backward_matches_finite_differences():
    grid, shapes, tail, rho = (2, 8, 20), [(1, 8, 16)], 0, [(1, 2)]
    q, k, v, g, out = _case(grid, shapes, tail, 5, rho)
    slots, nv, lists = out["slots"], out["n_valid"], out["lists"]
    qt, kt, vt = out["q_tiled"], out["k_tiled"], out["v_tiled"]
    dot = O.permute(g, slots)
    dq, dk, dv = O.attention_backward(qt, kt, vt, nv, lists, SCALE, np.nan_to_num(out["o_tiled"]),
                                      out["lse"], dot)

    def loss(qt_, kt_, vt_):
        o, _ = O.attention(qt_, kt_, vt_, nv, lists, SCALE)
        return float((np.nan_to_num(o) * dot).sum())

    rng = np.random.default_rng(1)
    eps = 1e-5
    valid_rows = np.flatnonzero(slots[0] >= 0)
    for which, grad in ((0, dq), (1, dk), (2, dv)):
        for _ in range(6):
            r = int(rng.choice(valid_rows))
            d = int(rng.integers(128))
            xs = [qt.copy(), kt.copy(), vt.copy()]
            xs[which][0, 0, r, d] += eps
            up = loss(*xs)
            xs[which][0, 0, r, d] -= 2 * eps
            dn = loss(*xs)
            fd = (up - dn) / (2 * eps)
            assert fd == pytest.approx(grad[0, 0, r, d], rel=1e-5, abs=1e-8), (which, r, d)


def test_transposed_lists_and_a_planted_mistake():
    q, k, v, g, out = _case((3, 9, 20), [(1, 8, 16), (2, 8, 8)], 0, 2, [(1, 3)])
    lists, nTh = out["lists"], out["nT_per_head"]
    nT = out["q_tiled"].shape[2] // 128
    T = O.transpose_lists(lists, nTh, nT)
    for h in range(len(nTh)):
        for i in range(nTh[h]):
            row = set(np.concatenate([lists.full[0][h][i], lists.partial[0][h][i]]).tolist())
            for j in range(nT):
                assert (j in row) == (i in set(T[0][h][j].tolist()))
        for j in range(nT):
            assert np.all(np.diff(T[0][h][j]) > 0)
    # a dropped entry makes the transposed lists disagree with the forward lists
    bad = O.BlockLists([[[r for r in hh] for hh in lists.full[0]]], lists.partial)
    i = 2
    bad.full[0][0][i] = bad.full[0][0][i][1:]
    Tb = O.transpose_lists(bad, nTh, nT)
    assert any(not np.array_equal(a, b) for a, b in zip(Tb[0][0], T[0][0]))
