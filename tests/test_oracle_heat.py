"""Pins of the oracle's block heat and mask-quality functions (no GPU).

* heat equals the block sums of a library softmax over the dense raster scores, taken
  through the tile map's token ownership (an independent route: no tiled layout);
* every valid row of heat sums to 1; rows past a head's tile count are 0;
* a hand-worked example fixes the attention-mass weighting and the recall definition;
* the full mask keeps all of the mass; the oracle mask keeps at least as much mass in
  every row as any other mask with the same budgets that contains the diagonal, and has
  recall 1 against itself; a planted mistake (one row's mask shifted) lowers recall.
"""
import numpy as np
import pytest
import torch

from oracle import veda_oracle as O

SCALE = 1.0 / np.sqrt(128)


def _case(grid, shapes, tail, seed, B=1):
    H = len(shapes)
    N = grid[0] * grid[1] * grid[2] + tail
    rng = np.random.default_rng(seed)
    q, k = rng.standard_normal((2, B, N, H, 128))
    k[..., :] += 0.5 * q[..., :]           # some correlation, so the heat is far from uniform
    maps = [O.tile_map(grid, tuple(shapes[h]), tail) for h in range(H)]
    nT_per_head = [len(m.n_valid) for m in maps]
    slots, n_valid, segment = O.stack_maps(maps)
    return q, k, slots, n_valid, segment, nT_per_head


@pytest.mark.parametrize("grid,shapes,tail", [
    ((2, 8, 20), [(1, 8, 16)], 0),                  # partial tiles along w
    ((3, 9, 20), [(1, 8, 16), (2, 8, 8)], 0),       # two shapes, padded grid
    ((2, 8, 12), [(4, 4, 8)], 77),                  # tail tokens (a second segment)
])
def test_heat_equals_block_sums_of_library_softmax(grid, shapes, tail):
    q, k, slots, n_valid, segment, nT_per_head = _case(grid, shapes, tail, 5)
    heat = O.block_heat(O.permute(q, slots), O.permute(k, slots), n_valid, nT_per_head, SCALE)
    B, N, H, _ = q.shape
    for h in range(H):
        tile_of = np.full(N, -1)
        for s in np.flatnonzero(slots[h] >= 0):
            tile_of[slots[h, s]] = s // 128
        P = torch.softmax(SCALE * torch.from_numpy(q[0, :, h]) @ torch.from_numpy(k[0, :, h]).T, dim=1).numpy()
        n = nT_per_head[h]
        for i in range(n):
            rows = tile_of == i
            expect = np.array([P[rows][:, tile_of == j].sum(axis=1).mean() for j in range(n)])
            assert np.allclose(heat[0, h, i, :n], expect, rtol=1e-12, atol=1e-14)
        assert np.allclose(heat[0, h, :n, :n].sum(axis=1), 1.0, atol=1e-12)
        assert not heat[0, h, n:].any()


def _lists(rows_full, rows_part):
    return O.BlockLists([[[np.array(r, np.int64) for r in rows_full]]],
                        [[[np.array(r, np.int64) for r in rows_part]]])


def test_mask_quality_hand_example():
    heat = np.array([[[[0.5, 0.3, 0.2],
                       [0.1, 0.6, 0.3],
                       [0.0, 0.25, 0.75]]]])
    n_valid = np.array([[128, 64, 32]])
    pred = _lists([[0], [1], []], [[2], [], [2]])          # row sets {0,2}, {1}, {2}
    orac = _lists([[0, 1], [1], []], [[], [2], [2]])       # row sets {0,1}, {1,2}, {2}
    mass_rows, recall_rows, mass, recall = O.mask_quality(heat, n_valid, [3], pred, orac)
    assert np.allclose(mass_rows[0, 0], [0.7, 0.6, 0.75])
    assert np.allclose(recall_rows[0, 0], [0.5, 0.5, 1.0])
    assert mass == pytest.approx((128 * 0.7 + 64 * 0.6 + 32 * 0.75) / 224)
    assert recall == pytest.approx(2.0 / 3.0)


def test_oracle_mask_keeps_the_most_mass():
    q, k, slots, n_valid, segment, nT_per_head = _case((3, 9, 20), [(1, 8, 16), (2, 8, 8)], 0, 9)
    heat = O.block_heat(O.permute(q, slots), O.permute(k, slots), n_valid, nT_per_head, SCALE)
    rho = [(1, 3)]
    oracle = O.select(heat, n_valid, segment, nT_per_head, rho)
    full = O.select(heat, n_valid, segment, nT_per_head, [(1, 1)])
    m_full = O.mask_quality(heat, n_valid, nT_per_head, full, oracle)
    assert m_full[2] == pytest.approx(1.0, abs=1e-12) and m_full[3] == pytest.approx(1.0)
    m_or = O.mask_quality(heat, n_valid, nT_per_head, oracle, oracle)
    assert m_or[3] == pytest.approx(1.0)
    rng = np.random.default_rng(3)
    H = heat.shape[1]
    for _ in range(5):
        full_rows, part_rows = [[]], [[]]
        fr, pr = [], []
        for h in range(H):
            n = nT_per_head[h]
            f_h, p_h = [], []
            for i in range(n):
                kk = len(oracle.full[0][h][i]) + len(oracle.partial[0][h][i])
                pick = np.sort(np.concatenate([[i], rng.choice(np.delete(np.arange(n), i), kk - 1, replace=False)]))
                f_h.append(pick[n_valid[h, pick] == 128])
                p_h.append(pick[n_valid[h, pick] < 128])
            f_h += [np.zeros(0, np.int64)] * (heat.shape[2] - n)
            p_h += [np.zeros(0, np.int64)] * (heat.shape[2] - n)
            fr.append(f_h)
            pr.append(p_h)
        rand = O.BlockLists([fr], [pr])
        m_rand = O.mask_quality(heat, n_valid, nT_per_head, rand, oracle)
        assert np.all(m_or[0] >= m_rand[0] - 1e-12)
        assert m_rand[3] < 1.0
    # a planted mistake: one row of the oracle mask shifted by one tile loses recall
    bad_full = [[list(r) for r in oracle.full[0][h]] for h in range(H)]
    bad_part = [[list(r) for r in oracle.partial[0][h]] for h in range(H)]
    i = 3
    shifted = sorted({(x + 1) % nT_per_head[0] for x in bad_full[0][i] + bad_part[0][i]})
    bad_full[0][i] = [x for x in shifted if n_valid[0, x] == 128]
    bad_part[0][i] = [x for x in shifted if n_valid[0, x] < 128]
    bad = O.BlockLists([[[np.array(r, np.int64) for r in hr] for hr in bad_full]],
                       [[[np.array(r, np.int64) for r in hr] for hr in bad_part]])
    assert O.mask_quality(heat, n_valid, nT_per_head, bad, oracle)[3] < 1.0
