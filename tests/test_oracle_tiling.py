"""Pins of the oracle's tile map, permute and unpermute (no GPU).

The tile map is checked against a hand-derived fixture, against an independent
vectorised construction (pad, reshape, transpose, compact), and against the
tile counts the workloads' grids imply.
"""
import os

import numpy as np
import pytest

import synth
from oracle import veda_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _parse_ranges(spec):
    out = []
    for part in spec.split():
        a, b = part.split("-")
        out.extend(range(int(a), int(b) + 1))
    return out


def _reshape_map(grid, shape):
    """Independent construction: pad the index grid with -1, cut it into tiles by
    reshape/transpose, and move each tile's valid entries to its front (stable)."""
    T, Hg, Wg = grid
    tt, th, tw = shape
    idx = np.arange(T * Hg * Wg).reshape(T, Hg, Wg)
    Tp, Hp, Wp = -(-T // tt) * tt, -(-Hg // th) * th, -(-Wg // tw) * tw
    pad = np.full((Tp, Hp, Wp), -1)
    pad[:T, :Hg, :Wg] = idx
    t = pad.reshape(Tp // tt, tt, Hp // th, th, Wp // tw, tw).transpose(0, 2, 4, 1, 3, 5)
    t = t.reshape(-1, tt * th * tw)
    out = []
    for row in t:
        v = row[row >= 0]
        out.append(np.concatenate([v, np.full(len(row) - len(v), -1)]))
    return np.concatenate(out)


def test_hand_fixture_1x8x20():
    m = O.tile_map((1, 8, 20), (1, 8, 16))
    lines = [l for l in open(os.path.join(GOLDEN, "tilemap_1x8x20_t1x8x16.txt")) if l.startswith("tile")]
    assert len(lines) == len(m.n_valid) == 2
    for line in lines:
        head, spec = line.split(":")
        _, i, _, n = head.split()
        i, n = int(i), int(n)
        toks = _parse_ranges(spec)
        assert m.n_valid[i] == n == len(toks)
        assert list(m.slots[i * 128:i * 128 + n]) == toks
        assert (m.slots[i * 128 + n:(i + 1) * 128] == -1).all()


def test_tiny_workload_is_frame_per_tile():
    # one tile = one 8x16 frame: the slot order is the raster order itself
    m = O.tile_map((4, 8, 16), (1, 8, 16))
    assert (m.slots == np.arange(512)).all()
    assert (m.n_valid == 128).all() and (m.segment == 0).all()


@pytest.mark.parametrize("grid,shape", [
    ((3, 5, 9), (2, 8, 8)), ((31, 30, 54), (1, 8, 16)), ((16, 32, 56), (4, 4, 8)),
    ((8, 32, 32), (2, 8, 8)), ((5, 13, 7), (4, 4, 8)), ((1, 1, 1), (1, 8, 16))])
def test_matches_reshape_construction(grid, shape):
    m = O.tile_map(grid, shape)
    assert (m.slots == _reshape_map(grid, shape)).all()


@pytest.mark.parametrize("w,nT,Npad,N", [
    (synth.TINY, 4, 512, 512), (synth.SMALL, 64, 8192, 8192),
    (synth.CLIP16x9, 496, 63488, 50220), (synth.MIXED, 229, 29312, 29312)])
def test_workload_tile_counts(w, nT, Npad, N):
    for shape in set(w.head_shapes):
        m = O.tile_map(w.grid, shape, w.n_tail)
        assert len(m.n_valid) == nT
        assert int(m.n_valid.sum()) == N
    assert w.nT == nT and w.Npad == Npad and w.N == N


@pytest.mark.parametrize("T,nT", [(5, 80), (15, 240), (31, 496), (62, 992)])
def test_length_sweep_tile_counts(T, nT):
    m = O.tile_map((T, 30, 54), (1, 8, 16))
    assert len(m.n_valid) == nT


def test_bijection_and_valid_prefix():
    for grid, shape, tail in [((3, 5, 9), (2, 8, 8), 0), ((16, 32, 56), (4, 4, 8), 640),
                              ((7, 9, 11), (1, 8, 16), 200)]:
        m = O.tile_map(grid, shape, tail)
        N = grid[0] * grid[1] * grid[2] + tail
        valid = m.slots[m.slots >= 0]
        assert sorted(valid.tolist()) == list(range(N))        # every token exactly once
        s = m.slots.reshape(-1, 128)
        for i, row in enumerate(s):                            # pads only at the tile's end
            n = int((row >= 0).sum())
            assert n == m.n_valid[i] >= 1
            assert (row[:n] >= 0).all() and (row[n:] == -1).all()


def test_tail_tiles_and_segments():
    m = O.tile_map((16, 32, 56), (2, 8, 8), 640)
    assert (m.segment[:224] == 0).all() and (m.segment[224:] == 1).all()
    assert (m.slots[224 * 128:229 * 128] == np.arange(28672, 28672 + 640)).all()
    m2 = O.tile_map((2, 8, 16), (1, 8, 16), 130)             # ragged last tail tile
    assert list(m2.n_valid) == [128, 128, 128, 2]
    assert list(m2.slots[3 * 128:3 * 128 + 3]) == [256 + 128, 256 + 129, -1]


def test_tile_order_reorders_video_tiles_only():
    base = O.tile_map((16, 32, 56), (4, 4, 8), 640)
    order = np.random.default_rng(0).permutation(224)
    m = O.tile_map((16, 32, 56), (4, 4, 8), 640, order)
    for p, i in enumerate(order):
        assert (m.slots[p * 128:(p + 1) * 128] == base.slots[i * 128:(i + 1) * 128]).all()
    assert (m.slots[224 * 128:] == base.slots[224 * 128:]).all()
    with pytest.raises(ValueError):
        O.tile_map((16, 32, 56), (4, 4, 8), 640, np.zeros(224, dtype=int))


def test_bad_tile_shape_rejected():
    with pytest.raises(ValueError):
        O.tile_map((4, 8, 16), (2, 8, 16))


def test_permute_unpermute_identity_and_zero_pads():
    rng = np.random.default_rng(1)
    grid, tail = (3, 5, 9), 20
    maps = [O.tile_map(grid, (2, 8, 8), tail), O.tile_map(grid, (4, 4, 8), tail,
                                                           rng.permutation(4))]
    slots, n_valid, seg = O.stack_maps(maps)
    N = 135 + tail
    x = rng.standard_normal((2, N, 2, 128))
    xt = O.permute(x, slots)
    for h in range(2):
        assert (xt[:, h][:, slots[h] < 0] == 0).all()
        for s in np.flatnonzero(slots[h] >= 0)[:50]:
            assert (xt[:, h, s] == x[:, slots[h, s], h]).all()
    assert (O.unpermute(xt, slots, N) == x).all()
