"""Seeded synthetic inputs and the workload table for the Veda sparse-attention path.

This module holds no step of the method. It only draws the random inputs that
both sides of every parity check consume -- Q, K, V, the per-head projection
weights and the per-head tile orders -- and names the workloads they are drawn
for. The oracle (``oracle/``) and the CUDA library never import each other; tests
and the benchmark feed both from here, so both see identical bytes.

Recipe (the pages' workloads are real MiniMax-H3 clips that are not available,
so these stand in for them with the pages' shapes):

* Q, K, V are ``[B, N, H, D]`` raster-order tensors, rounded once to bf16.
* "iid" workloads: Q, K, V ~ N(0, 1).
* "field" workloads: one smoothed field F per (batch, head, channel) -- N(0,1)
  noise filtered by a separable Gaussian (sigma 2 tokens, truncated at 3 sigma,
  half-sample-symmetric "reflect" boundary) along t, h and w of the video grid,
  and along the sequence for the appended 1D tail tokens -- normalised to unit
  standard deviation per channel. Q = F + 0.5 N1, K = F + 0.5 N2 with
  independent noise, V ~ N(0, 1).
* Projection weights W_q, W_k: fp32 ``[H, D, 3D]`` ~ N(0, 0.02).
* Per-head tile orders (workloads with ``shuffle_heads``): a seeded random
  permutation of each head's video tiles.

Seeds: torch's CPU generator (``torch.Generator().manual_seed``), seed = 1000 * workload id + tensor id (Q field 1, Q noise 2,
K noise 3, V 4, W_q 5, W_k 6, tile orders 7); the tiny workload uses seed 0
for all of Q, K and V (drawn in that order from one generator).
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence, Tuple

import numpy as np
import scipy.ndimage
import torch

D_HEAD = 128
TILE_TOKENS = 128


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: geometry, budgets and input recipe."""

    name: str
    wid: int                      # workload id, used in the seeds
    B: int
    H: int
    grid: Tuple[int, int, int]    # video grid (T, Hg, Wg)
    head_shapes: Tuple[Tuple[int, int, int], ...]  # one (t, h, w) tile per head
    n_tail: int = 0               # appended 1D (audio) tokens
    rho: Tuple[Tuple[int, int], ...] = ((1, 10),)   # density per key segment
    field: bool = True            # smoothed field (else iid normal)
    shuffle_heads: bool = False   # per-head random tile order
    D: int = D_HEAD

    @property
    def n_video(self) -> int:
        T, Hg, Wg = self.grid
        return T * Hg * Wg

    @property
    def N(self) -> int:
        return self.n_video + self.n_tail

    def video_tiles(self, shape: Tuple[int, int, int]) -> int:
        T, Hg, Wg = self.grid
        tt, th, tw = shape
        if self.n_video == 0:
            return 0
        return math.ceil(T / tt) * math.ceil(Hg / th) * math.ceil(Wg / tw)

    def tiles_per_head(self) -> List[int]:
        tail = math.ceil(self.n_tail / TILE_TOKENS)
        return [self.video_tiles(s) + tail for s in self.head_shapes]

    @property
    def nT(self) -> int:
        return max(self.tiles_per_head())

    @property
    def Npad(self) -> int:
        return self.nT * TILE_TOKENS

    @property
    def n_segments(self) -> int:
        return len(self.rho)

    def with_rho(self, rho: Sequence[Tuple[int, int]], name: Optional[str] = None) -> "Workload":
        return dataclasses.replace(self, rho=tuple(tuple(r) for r in rho),
                                   name=name or self.name)


def _uniform(H, shape):
    return tuple([tuple(shape)] * H)


TINY = Workload("tiny", 1, B=1, H=2, grid=(4, 8, 16), head_shapes=_uniform(2, (1, 8, 16)),
                rho=((1, 2),), field=False)
SMALL = Workload("small", 2, B=1, H=8, grid=(8, 32, 32), head_shapes=_uniform(8, (2, 8, 8)))
CLIP16x9 = Workload("clip16x9", 3, B=1, H=40, grid=(31, 30, 54),
                    head_shapes=_uniform(40, (1, 8, 16)))
MIXED = Workload("mixed", 4, B=1, H=32, grid=(16, 32, 56),
                 head_shapes=tuple([(2, 8, 8)] * 16 + [(4, 4, 8)] * 16), n_tail=640,
                 rho=((1, 10), (1, 10)), shuffle_heads=True)

SWEEP_DENSITIES = ((1, 20), (1, 10), (1, 5), (1, 2), (1, 1))
SWEEP_FRAMES = (5, 15, 31, 62)


def sweep_density(p: int, q: int) -> Workload:
    return dataclasses.replace(CLIP16x9, name=f"clip16x9_rho{p}_{q}", wid=5, rho=((p, q),))


def sweep_length(T: int) -> Workload:
    return dataclasses.replace(CLIP16x9, name=f"len_T{T}", wid=5, grid=(T, 30, 54))


WORKLOADS = {w.name: w for w in (TINY, SMALL, CLIP16x9, MIXED)}


def get(name: str) -> Workload:
    if name in WORKLOADS:
        return WORKLOADS[name]
    if name.startswith("clip16x9_rho"):
        p, q = name[len("clip16x9_rho"):].split("_")
        return sweep_density(int(p), int(q))
    if name.startswith("len_T"):
        return sweep_length(int(name[len("len_T"):]))
    raise KeyError(name)


# --------------------------------------------------------------------------------------
# random draws
# --------------------------------------------------------------------------------------

class _Rng:
    """Seeded normal draws (torch's CPU Mersenne-Twister generator: fast and reproducible)."""

    def __init__(self, seed: int):
        self.g = torch.Generator().manual_seed(seed)

    def standard_normal(self, shape, dtype=np.float32) -> np.ndarray:
        return torch.randn(tuple(shape), generator=self.g, dtype=torch.float32).numpy()

    def permutation(self, n: int) -> np.ndarray:
        return torch.randperm(n, generator=self.g).numpy()


def _rng(seed: int) -> _Rng:
    return _Rng(seed)


def _gauss_kernel(sigma: float = 2.0, truncate: float = 3.0) -> np.ndarray:
    r = int(truncate * sigma + 0.5)
    x = np.arange(-r, r + 1, dtype=np.float64)
    k = np.exp(-0.5 * (x / sigma) ** 2)
    return (k / k.sum()).astype(np.float32)


def _smooth_axis(a: np.ndarray, axis: int, k: np.ndarray) -> np.ndarray:
    """Separable Gaussian along one axis, half-sample-symmetric reflection at both ends."""
    if a.shape[axis] == 0:
        return a
    return scipy.ndimage.correlate1d(a, k, axis=axis, mode="reflect")


def _field(rng: "_Rng", B: int, grid, n_tail: int, heads: Sequence[int], D: int) -> np.ndarray:
    """Unit-std smoothed field, shape [B, N, len(heads), D], fp32."""
    T, Hg, Wg = grid
    k = _gauss_kernel()
    nh = len(heads)
    nv = T * Hg * Wg
    out = np.empty((B, nv + n_tail, nh, D), dtype=np.float32)
    for b in range(B):
        if nv:
            f = rng.standard_normal((T, Hg, Wg, nh, D), dtype=np.float32)
            for h0 in range(0, nh, 4):          # smooth a few heads at a time (memory)
                c = np.ascontiguousarray(f[:, :, :, h0:h0 + 4])
                for ax in range(3):
                    c = _smooth_axis(c, ax, k)
                c = c.reshape(nv, -1, D)
                c /= np.maximum(c.std(axis=0, keepdims=True), 1e-6)
                out[b, :nv, h0:h0 + 4] = c
            del f
        if n_tail:
            g = rng.standard_normal((n_tail, nh, D), dtype=np.float32)
            g = _smooth_axis(g, 0, k)
            g /= np.maximum(g.std(axis=0, keepdims=True), 1e-6)
            out[b, nv:] = g
    return out


def _to_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16)


@dataclasses.dataclass
class Inputs:
    """Raster-order inputs for one workload (CPU tensors)."""

    q: torch.Tensor          # [B, N, H, D] bf16
    k: torch.Tensor
    v: torch.Tensor
    wq: torch.Tensor         # [H, D, 3D] fp32
    wk: torch.Tensor
    tile_order: Optional[np.ndarray]  # [H, nT] int32 (first n_video_tiles entries used) or None


def make_inputs(w: Workload, heads: Optional[Sequence[int]] = None) -> Inputs:
    """Draw the seeded inputs of workload ``w`` (optionally only some heads' slices).

    Drawing a subset of heads gives the same values as slicing the full draw only
    for iid workloads; field workloads draw per head block, so callers that need a
    subset for parity always draw the same subset on both sides.
    """
    B, N, H, D = w.B, w.N, w.H, w.D
    hs = list(range(H)) if heads is None else list(heads)
    if not w.field:
        g = _rng(0 if w.wid == 1 else 1000 * w.wid + 1)
        q = g.standard_normal((B, N, H, D), dtype=np.float32)
        k = g.standard_normal((B, N, H, D), dtype=np.float32)
        v = g.standard_normal((B, N, H, D), dtype=np.float32)
        q, k, v = q[:, :, hs], k[:, :, hs], v[:, :, hs]
    else:
        F = _field(_rng(1000 * w.wid + 1), B, w.grid, w.n_tail, hs, D)
        q = _rng(1000 * w.wid + 2).standard_normal(F.shape, dtype=np.float32)
        q *= 0.5
        q += F
        k = _rng(1000 * w.wid + 3).standard_normal(F.shape, dtype=np.float32)
        k *= 0.5
        k += F
        del F
        v = _rng(1000 * w.wid + 4).standard_normal((B, N, len(hs), D), dtype=np.float32)
    wq = (0.02 * _rng(1000 * w.wid + 5).standard_normal((H, D, 3 * D), dtype=np.float32))[hs]
    wk = (0.02 * _rng(1000 * w.wid + 6).standard_normal((H, D, 3 * D), dtype=np.float32))[hs]
    order = tile_orders(w)
    if order is not None:
        order = order[hs]
    return Inputs(_to_bf16(q), _to_bf16(k), _to_bf16(v),
                  torch.from_numpy(np.ascontiguousarray(wq)),
                  torch.from_numpy(np.ascontiguousarray(wk)), order)


def tile_orders(w: Workload) -> Optional[np.ndarray]:
    """Seeded per-head tile orders [H, nT] (first n_video_tiles entries used), or None."""
    if not w.shuffle_heads:
        return None
    g = _rng(1000 * w.wid + 7)
    order = np.full((w.H, w.nT), -1, dtype=np.int32)
    for h in range(w.H):
        nv = w.video_tiles(w.head_shapes[h])
        order[h, :nv] = g.permutation(nv).astype(np.int32)
    return order


def head_subset(w: Workload, heads: Sequence[int]) -> Workload:
    """The same workload restricted to some heads (shapes follow the heads)."""
    return dataclasses.replace(w, H=len(heads), head_shapes=tuple(w.head_shapes[h] for h in heads))


def random_lists(rng: np.random.Generator, nT: int, blocks_per_row: Sequence[int]):
    """Uniform random block sets with a forced diagonal, for 'new pattern per call' timing.

    Returns sorted int32 arrays per row. This is an input recipe for timing only
    (the predicted lists come from the method's own selection stage).
    """
    rows = []
    for r, kr in enumerate(blocks_per_row):
        others = np.delete(np.arange(nT), r)
        pick = rng.choice(others, size=max(0, min(kr, nT) - 1), replace=False)
        rows.append(np.sort(np.concatenate([[r], pick])).astype(np.int32))
    return rows

