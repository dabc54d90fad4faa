"""GPU parity of the oracle tile-plan search (the library's calls chained per candidate shape).

Both sides search the same seeded bf16 inputs over the same candidate shapes: the GPU with
its own heat, oracle masks and sparse attention, the oracle in fp64. Tolerance (derived):
the error of a shape is a ratio of sums of squares of output differences that are ~0.1 of
the output or more, while the GPU's outputs carry bf16 rounding (2^-9 relative) and its
oracle masks may differ from the fp64 ones at near-ties of the heat, so per-entry agreement
within 5% relative. The vote itself is compared twice: on the GPU's own errors against the
oracle's vote of the same errors (identical inputs, identical plan), and, on heads built so
that each has one clearly best shape, against the oracle's plan from its own errors.
"""
import numpy as np
import pytest
import torch

from oracle import veda_oracle as O
import parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
CANDIDATES = [(1, 8, 16), (2, 8, 8), (4, 4, 8), (2, 4, 16)]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from block_sparse_attention_max_b200 import build
    build.build()
    V = P.veda()
    V.lib()
    yield
    V.check_device_status()


def test_tile_plan_search_matches_oracle():
    from block_sparse_attention_max_b200 import plan
    grid, H, rho = (4, 16, 32), 3, [(1, 4)]
    N = grid[0] * grid[1] * grid[2]
    gen = torch.Generator().manual_seed(9008)
    q, k, v = (torch.randn((1, N, H, 128), generator=gen) for _ in range(3))
    # heads with different structure: keys correlated with the queries to different degrees
    for h, a in enumerate((0.4, 0.8, 1.2)):
        k[:, :, h] += a * q[:, :, h]
    q, k, v = (t.to(torch.bfloat16) for t in (q, k, v))
    res = plan.tile_plan_search(q.to(DEV), k.to(DEV), v.to(DEV), grid, 0, CANDIDATES, rho, P.SCALE)
    err_o = O.shape_errors(P.f64(q), P.f64(k), P.f64(v), grid, 0, CANDIDATES, rho, P.SCALE)
    assert np.all(np.abs(res.errors - err_o) <= 0.05 * err_o), (res.errors, err_o)
    # the vote on the GPU's errors is the oracle's vote of the same errors
    kept_o, assign_o = O.tile_plan(res.errors)
    assert res.kept == list(kept_o) and res.assign.tolist() == assign_o.tolist()
    assert len(res.kept) <= 2 and set(res.assign.tolist()) <= set(res.kept)


def _axis_field(grid, varying, gen):
    """One N(0,1) vector per coordinate of the `varying` axes ('t', 'h', 'w'), constant along
    the others: tokens that agree on the varying coordinates hold the same vector."""
    T, Hg, Wg = grid
    sizes = [T if "t" in varying else 1, Hg if "h" in varying else 1, Wg if "w" in varying else 1]
    f = torch.randn(sizes + [128], generator=gen)
    return f.expand(T, Hg, Wg, 128).reshape(T * Hg * Wg, 128)


def test_tile_plan_search_picks_each_heads_shape():
    """Heads whose queries and keys vary along one axis only. A query then attends (almost
    only) to the keys that share its coordinate on that axis, and the shape whose tiles hold
    most of those keys in the fewest tiles loses least under a budget of two key tiles per
    row (16x more keys than one tile holds):
      head 0 varies along t (8 frames): (1, 8, 16) tiles cover a frame in 4 tiles, so two
             tiles keep 1/2 of a query's keys; (2, 8, 8): 1/4; (4, 4, 8): 1/8; (8, 4, 4): 1/16;
      heads 1, 2 vary along w (32 columns): (8, 4, 4) covers a 4-column group in 4 tiles,
             so 1/2; (2, 8, 8) and (4, 4, 8): 1/4; (1, 8, 16): 1/8.
    With uniform weights over m keys and V ~ N(0, 1), keeping a fraction f gives a relative
    output error of (1 - f) / f: 1, 3, 7, 15, so every head's best shape wins by 3x. The
    layer keeps {(1, 8, 16), (8, 4, 4)} (two votes for the latter, one for the former), or
    only (8, 4, 4) when one shape is allowed."""
    from block_sparse_attention_max_b200 import plan
    grid, rho = (8, 16, 32), [(1, 16)]
    cands = [(1, 8, 16), (4, 4, 8), (2, 8, 8), (8, 4, 4)]
    gen = torch.Generator().manual_seed(9010)
    q = torch.stack([_axis_field(grid, "t", gen), _axis_field(grid, "w", gen), _axis_field(grid, "w", gen)],
                    dim=1)[None]
    k = q + 0.05 * torch.randn(q.shape, generator=gen)
    v = torch.randn(q.shape, generator=gen)
    q, k, v = (t.to(torch.bfloat16) for t in (q, k, v))
    err_o = O.shape_errors(P.f64(q), P.f64(k), P.f64(v), grid, 0, cands, rho, P.SCALE)
    best = np.sort(err_o, axis=1)
    assert (best[:, 1] > 2.5 * best[:, 0]).all(), err_o          # the construction separates the shapes
    for ms, kept_want, assign_want in ((2, [0, 3], [0, 3, 3]), (1, [3], [3, 3, 3])):
        res = plan.tile_plan_search(q.to(DEV), k.to(DEV), v.to(DEV), grid, 0, cands, rho, P.SCALE,
                                    max_shapes=ms)
        assert np.all(np.abs(res.errors - err_o) <= 0.05 * err_o), (res.errors, err_o)
        kept_o, assign_o = O.tile_plan(err_o, ms)
        assert list(kept_o) == kept_want and assign_o.tolist() == assign_want
        assert res.kept == kept_want and res.assign.tolist() == assign_want
        assert res.head_shapes() == [cands[c] for c in assign_want]
