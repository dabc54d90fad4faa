"""Oracle tile-plan search on the GPU: the library's calls chained per candidate tile shape.

"Miowtion" README, Key Features / Veda sparse attention: "oracle tile-plan search (relative
output MSE under the best mask), majority vote, at most two shapes per layer". For every
candidate (t, h, w) tile shape this runs, on the GPU, the permute, dense attention for the
LSE, the block heat, the oracle mask (the selection step on the heat), block-sparse
attention with that mask and the unpermute, and takes each head's relative output error
against dense attention (veda_rel_error). Each head votes for its lowest-error shape; the
layer keeps the (at most) two most voted shapes (ties to the earlier candidate) and every
head takes the better of the kept shapes for it.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence, Tuple

import numpy as np
import torch

from . import veda as V


@dataclasses.dataclass
class TilePlan:
    candidates: List[Tuple[int, int, int]]
    errors: np.ndarray          # [H, C] relative output error of each shape under its best mask
    kept: List[int]             # candidate indices the layer keeps
    assign: np.ndarray          # [H] candidate index per head

    def head_shapes(self) -> List[Tuple[int, int, int]]:
        return [self.candidates[c] for c in self.assign]


def shape_errors(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, grid: Tuple[int, int, int], n_tail: int,
                 candidates: Sequence[Tuple[int, int, int]], rho: Sequence[Tuple[int, int]],
                 scale: float) -> np.ndarray:
    """[H, C] relative output error of every candidate shape under its heat-oracle mask."""
    B, N, H, D = q.shape
    dev = q.device
    o_dense = None
    sums = []
    for shape in candidates:
        maps = V.build_tile_map(grid, [tuple(shape)] * H, n_tail).to(dev)
        qt, kt, vt = V.permute_tiles(q, maps), V.permute_tiles(k, maps), V.permute_tiles(v, maps)
        nT = maps.nT
        dense = V.select_blocks(torch.zeros((B, H, nT, nT), dtype=torch.float32, device=dev), maps,
                                [(1, 1)] * len(rho))
        o_t, lse = V.block_sparse_attn_fwd(qt, kt, vt, maps, dense, scale)
        if o_dense is None:
            o_dense = V.unpermute(o_t, maps, N)      # dense attention does not depend on the tiling
        heat = V.block_heat(qt, kt, maps, dense, lse, scale)
        mask = V.select_blocks(heat, maps, rho)
        o_s, _ = V.block_sparse_attn_fwd(qt, kt, vt, maps, mask, scale, want_lse=False)
        sums.append(V.rel_error(V.unpermute(o_s, maps, N), o_dense))
    V.check_device_status()
    s = torch.stack(sums, dim=1).double().cpu().numpy()     # [H, C, 2]
    return s[..., 0] / s[..., 1]


def tile_plan_search(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, grid: Tuple[int, int, int],
                     n_tail: int, candidates: Sequence[Tuple[int, int, int]], rho: Sequence[Tuple[int, int]],
                     scale: float, max_shapes: int = 2) -> TilePlan:
    err = shape_errors(q, k, v, grid, n_tail, candidates, rho, scale)
    kept, assign = V.tile_plan_vote(err, max_shapes)
    return TilePlan(list(map(tuple, candidates)), err, kept, assign)
