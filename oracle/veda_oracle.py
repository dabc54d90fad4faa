"""Plain fp64 CPU oracle of the Veda block-sparse attention hot path (test infrastructure).

This module is test infrastructure only. It exists so that the CUDA library can be
checked against something written straight from the method's description; only
the tests, the smoke check and the benchmark's CPU-baseline leg may import it.
It shares no code with the CUDA path and imports nothing from it.

Sources (web pages, cited by title and section):

* [AGENTS] "Deploying this checkpoint" -- the deployment recipe of the
  Minimax-H3-T2VA-Veda-8NFE-600Step-Preview predictor (preamble; section 2
  "Per-architecture notes", SM90 and SM100 paragraphs; section 4 "Verifying a
  deployment"; section 6 "What this checkpoint is not").
* [README] "Miowtion" -- the project README (bullet "Sparse acceleration (Veda)";
  "Key Features", sub-list "Veda sparse attention"; "NEWS" 2026/09/23).

The pages give the steps in prose only; where they leave a step open the reading
taken here is stated in the function's docstring (readings R1..R23). Everything
is computed in float64 from the bf16-rounded inputs (exact upcast).

Steps, in the path's order:

1. ``tile_map``      -- 3D tiling with padded grid and valid-prefix tiles
2. ``permute``       -- gather raster tokens into tile order
3. ``pool``          -- mean / max / min per tile
4. ``scores``        -- per-head residual projection, tile-pair dot products
5. ``budgets`` + ``select`` -- Bresenham budgets, forced diagonal, top-k lists
6. ``attention``     -- softmax attention over the listed key tiles
7. ``unpermute``     -- scatter back to raster order
7b. ``transpose_lists`` + ``attention_backward`` -- gradients over the same lists
8. ``block_heat`` + ``mask_quality`` -- teacher block heat from dense attention, the
   attention mass a mask keeps and its recall against the oracle mask
9. ``shape_errors`` + ``tile_plan`` -- oracle tile-plan search over candidate tile shapes
10. ``quantize_fp8`` / ``dequantize_fp8`` (``e4m3_round``, ``e4m3_codes``, ``e4m3_value``) --
   the e4m3 tensors of the FP8 attention variant, whose attention is ``attention`` on the
   dequantised tensors

plus ``dense_attention_raster``, an independent dense routine used as a pin.
Parity status: every function here is pinned by a ``-m "not gpu"`` test
(tests/test_oracle_*.py); none is "parity unpinned".
"""
from __future__ import annotations

import math
from fractions import Fraction
from typing import List, NamedTuple, Optional, Sequence, Tuple

import numpy as np

TILE = 128          # tokens per tile ([README] "3D tiles of 128 tokens")


# ---------------------------------------------------------------------------------------
# 1. tile map
# ---------------------------------------------------------------------------------------

class TileMap(NamedTuple):
    slots: np.ndarray     # [nT*128] int64: raster token index per slot, -1 for a pad slot
    n_valid: np.ndarray   # [nT] int64: valid tokens per tile (they occupy slots [0, n_valid))
    segment: np.ndarray   # [nT] int64: 0 = video tile, 1 = appended 1D (tail) tile


def tile_map(grid: Tuple[int, int, int], shape: Tuple[int, int, int], n_tail: int = 0,
             tile_order: Optional[Sequence[int]] = None) -> TileMap:
    """Slot -> raster-token map of one head.

    [README] bullet "Sparse acceleration (Veda)": video tokens are permuted into 3D
    tiles of 128 tokens. [README] Key Features / Veda sparse attention: up to two
    (t, h, w) tile shapes per layer (per head), padded grids with valid-prefix tiles,
    segmented reference/target budgets. [README] NEWS: per-head dynamic tile
    permutations.

    Readings:
      R1  the grid is padded up to a multiple of the tile shape on each axis; each
          tile lists its valid tokens first, in local (t, h, w) raster order, and its
          pad slots after them ("valid-prefix tiles").
      R2  tiles are enumerated in raster order of their tile coordinates; a raster
          token (t, h, w) has index t*Hg*Wg + h*Wg + w.
      R3  appended 1D (audio) tokens follow the video tokens in raster order (index
          T*Hg*Wg + j) and are cut into 1D tiles of 128, the last one valid-prefix
          padded; video tiles form key segment 0 and tail tiles segment 1.
      R4  a per-head tile permutation reorders the head's video tiles: position p
          holds the video tile ``tile_order[p]`` of the raster enumeration.
    """
    T, Hg, Wg = grid
    tt, th, tw = shape
    if tt * th * tw != TILE:
        raise ValueError(f"tile shape {shape} does not hold {TILE} tokens")
    tiles: List[List[int]] = []
    if T * Hg * Wg > 0:
        nt, nh, nw = -(-T // tt), -(-Hg // th), -(-Wg // tw)
        for it in range(nt):
            for ih in range(nh):
                for iw in range(nw):
                    toks = []
                    for lt in range(tt):
                        for lh in range(th):
                            for lw in range(tw):
                                t, h, w = it * tt + lt, ih * th + lh, iw * tw + lw
                                if t < T and h < Hg and w < Wg:
                                    toks.append((t * Hg + h) * Wg + w)
                    tiles.append(toks)
    n_video_tiles = len(tiles)
    if tile_order is not None:
        order = [int(i) for i in tile_order[:n_video_tiles]]
        if sorted(order) != list(range(n_video_tiles)):
            raise ValueError("tile_order is not a permutation of the video tiles")
        tiles = [tiles[i] for i in order]
    base = T * Hg * Wg
    for j0 in range(0, n_tail, TILE):
        tiles.append([base + j for j in range(j0, min(j0 + TILE, n_tail))])
    nT = len(tiles)
    slots = np.full(nT * TILE, -1, dtype=np.int64)
    n_valid = np.zeros(nT, dtype=np.int64)
    for i, toks in enumerate(tiles):
        slots[i * TILE:i * TILE + len(toks)] = toks
        n_valid[i] = len(toks)
    segment = np.array([0] * n_video_tiles + [1] * (nT - n_video_tiles), dtype=np.int64)
    return TileMap(slots, n_valid, segment)


def stack_maps(maps: Sequence[TileMap], nT: Optional[int] = None):
    """Per-head maps padded to a common tile count: slots [H, nT*128], n_valid/segment [H, nT].

    Tiles past a head's own count have n_valid 0 and all-pad slots.
    """
    nT = nT or max(len(m.n_valid) for m in maps)
    H = len(maps)
    slots = np.full((H, nT * TILE), -1, dtype=np.int64)
    n_valid = np.zeros((H, nT), dtype=np.int64)
    segment = np.zeros((H, nT), dtype=np.int64)
    for h, m in enumerate(maps):
        n = len(m.n_valid)
        slots[h, :n * TILE] = m.slots
        n_valid[h, :n] = m.n_valid
        segment[h, :n] = m.segment
    return slots, n_valid, segment


# ---------------------------------------------------------------------------------------
# 2. permute / 7. unpermute
# ---------------------------------------------------------------------------------------

def permute(x: np.ndarray, slots: np.ndarray) -> np.ndarray:
    """Gather raster tokens into tile order: out[b, h, s] = x[b, slots[h, s], h], 0 on pad slots.

    [README] "Sparse acceleration (Veda)": tokens are permuted into 3D tiles.
    x: [B, N, H, D]; slots: [H, Npad]. Returns [B, H, Npad, D] float64.
    """
    B, N, H, D = x.shape
    out = np.zeros((B, H, slots.shape[1], D), dtype=np.float64)
    for h in range(H):
        valid = slots[h] >= 0
        out[:, h, valid, :] = x[:, slots[h, valid], h, :]
    return out


def unpermute(o_tiled: np.ndarray, slots: np.ndarray, N: int) -> np.ndarray:
    """Inverse of ``permute`` on valid slots: out[b, slots[h, s], h] = o[b, h, s]; pad rows dropped.

    The attention output goes back to the raster order the rest of the model uses
    ([README] "Sparse acceleration (Veda)": only the attention runs on permuted
    tiles). o_tiled: [B, H, Npad, D]. Returns [B, N, H, D].
    """
    B, H, Npad, D = o_tiled.shape
    out = np.zeros((B, N, H, D), dtype=np.float64)
    for h in range(H):
        valid = slots[h] >= 0
        out[:, slots[h, valid], h, :] = o_tiled[:, h, valid, :]
    return out


# ---------------------------------------------------------------------------------------
# 3. pool
# ---------------------------------------------------------------------------------------

def pool(x_tiled: np.ndarray, n_valid: np.ndarray) -> np.ndarray:
    """Mean, max and min of each tile over its valid slots, per channel.

    [README] Key Features / Veda sparse attention: the predictor pools by
    mean/max/min. Reading R5: pooling runs over the tile's valid tokens only (pad
    slots are not data); a tile with no valid token (past a head's tile count)
    pools to zeros. x_tiled: [B, H, nT*128, D]; n_valid: [H, nT].
    Returns [B, H, nT, 3, D] with index 0 = mean, 1 = max, 2 = min.
    """
    B, H, Npad, D = x_tiled.shape
    nT = Npad // TILE
    out = np.zeros((B, H, nT, 3, D), dtype=np.float64)
    for h in range(H):
        for t in range(nT):
            n = int(n_valid[h, t])
            if n == 0:
                continue
            rows = x_tiled[:, h, t * TILE:t * TILE + n, :]
            out[:, h, t, 0] = rows.sum(axis=1) / n
            out[:, h, t, 1] = rows.max(axis=1)
            out[:, h, t, 2] = rows.min(axis=1)
    return out


# ---------------------------------------------------------------------------------------
# 4. scores
# ---------------------------------------------------------------------------------------

def project(pooled: np.ndarray, W: np.ndarray) -> np.ndarray:
    """Per-head residual projection: hat = mean + W_h [mean; max; min].

    [README] Key Features / Veda sparse attention: "mean/max/min pooling +
    per-head residual projection, 275M params". Reading R6: W_h is a D x 3D
    matrix per head, no bias, applied to the concatenated pooled features, and
    the residual is the mean; separate matrices for queries and keys. (Pinned by
    the parameter count: 2 * 128 * 384 per head over 56 heads and 50 blocks is
    275,251,200.) pooled: [B, H, nT, 3, D]; W: [H, D, 3D]. Returns [B, H, nT, D].
    """
    B, H, nT, _, D = pooled.shape
    f = pooled.reshape(B, H, nT, 3 * D)
    out = np.empty((B, H, nT, D), dtype=np.float64)
    for h in range(H):
        Wh = np.asarray(W[h], dtype=np.float64)
        out[:, h] = pooled[:, h, :, 0, :] + f[:, h] @ Wh.T
    return out


def scores(pooled_q: np.ndarray, pooled_k: np.ndarray, Wq: np.ndarray, Wk: np.ndarray) -> np.ndarray:
    """Score of every (query tile, key tile) pair: S[i, j] = qhat_i . khat_j.

    [README] "Sparse acceleration (Veda)": a small per-head predictor scores
    (query tile, key tile) pairs. Reading R7: the score is the plain dot product
    of the projected pooled features (no scale: a positive scale would not change
    the ranking). Returns [B, H, nT, nT].
    """
    qh = project(pooled_q, Wq)
    kh = project(pooled_k, Wk)
    return np.einsum("bhic,bhjc->bhij", qh, kh)


# ---------------------------------------------------------------------------------------
# 5. budgets and selection
# ---------------------------------------------------------------------------------------

def budgets(nT_head: int, segment: np.ndarray, rho: Sequence[Tuple[int, int]]) -> np.ndarray:
    """Blocks each query row takes from each key segment: k[r, s].

    [README] Key Features / Veda sparse attention: equal-kernel-cost budgets with
    Bresenham rounding, forced diagonal tiles, segmented reference/target budgets.

    Readings:
      R8  cost is counted in 128 x 128 kernel blocks; a segment s with nK_s key
          tiles and density rho_s = p/q gives row r (0-based, over the head's nT
          rows) k = floor((r+1) x) - floor(r x) with x = nK_s * rho_s taken exactly,
          so every row gets floor(x) or ceil(x) and the rows sum to floor(nT x).
      R9  the diagonal counts inside the budget of the query's own segment, which
          is raised to at least 1 so the diagonal always fits; every k is clamped
          to [0, nK_s].
    segment: [nT_head] segment of each tile. Returns int64 [nT_head, n_segments].
    """
    segment = np.asarray(segment[:nT_head])
    nseg = len(rho)
    k = np.zeros((nT_head, nseg), dtype=np.int64)
    for s, (p, q) in enumerate(rho):
        nK = int((segment == s).sum())
        x = Fraction(nK * p, q)
        for r in range(nT_head):
            k[r, s] = math.floor((r + 1) * x) - math.floor(r * x)
    for r in range(nT_head):
        own = int(segment[r])
        if own < nseg:
            k[r, own] = max(k[r, own], 1)
        for s in range(nseg):
            nK = int((segment == s).sum())
            k[r, s] = min(max(k[r, s], 0), nK)
    return k


class BlockLists(NamedTuple):
    full: List[List[List[np.ndarray]]]      # [B][H][nT] ascending key tiles with n_valid == 128
    partial: List[List[List[np.ndarray]]]   # [B][H][nT] ascending key tiles with n_valid < 128


def _canon(v: float) -> float:
    return 0.0 if v == 0.0 else float(v)      # -0 compares equal to +0


def select_row(S_row: np.ndarray, r: int, segment: np.ndarray, k_row: np.ndarray) -> np.ndarray:
    """Top-k key tiles of one query row, diagonal forced; ascending tile indices.

    [README] "Sparse acceleration (Veda)": only the top-scoring blocks are
    computed. [README] Key Features: forced diagonal tiles. Reading R10: within
    each key segment the k[s] best tiles are taken by score, highest first, equal
    scores going to the lower tile index (-0 equals +0); in the query's own
    segment the diagonal tile r is taken first and the other k-1 are the best of
    the rest. NaN scores are rejected. S_row, segment: [nT_head]; k_row: [n_seg].
    """
    nT = len(segment)
    if np.isnan(S_row[:nT]).any():
        raise ValueError("NaN score")
    chosen = []
    for s in range(len(k_row)):
        kk = int(k_row[s])
        cand = [j for j in range(nT) if segment[j] == s]
        if segment[r] == s and kk > 0:
            chosen.append(r)
            kk -= 1
            cand = [j for j in cand if j != r]
        cand.sort(key=lambda j: (-_canon(S_row[j]), j))
        chosen.extend(cand[:kk])
    return np.array(sorted(chosen), dtype=np.int64)


def select(S: np.ndarray, n_valid: np.ndarray, segment: np.ndarray, nT_per_head: Sequence[int],
           rho: Sequence[Tuple[int, int]]) -> BlockLists:
    """Block lists of every (batch, head, query row), split into full and partial tiles.

    [AGENTS] section 2, SM90 paragraph: the dense block mask is packed into
    full/partial index lists for the kernel. [README] Key Features: full/partial
    block lists, singleton mask_mod. Reading R11: a key tile is "full" when all
    128 of its slots are valid, "partial" otherwise (the kernel masks its pad
    slots); both lists are ascending. Rows past a head's tile count are empty.
    S: [B, H, nT, nT]; n_valid, segment: [H, nT].
    """
    B, H, nT, _ = S.shape
    full = [[[np.zeros(0, np.int64) for _ in range(nT)] for _ in range(H)] for _ in range(B)]
    part = [[[np.zeros(0, np.int64) for _ in range(nT)] for _ in range(H)] for _ in range(B)]
    for h in range(H):
        n = int(nT_per_head[h])
        seg = np.asarray(segment[h, :n])
        k = budgets(n, seg, rho)
        for b in range(B):
            for r in range(n):
                sel = select_row(S[b, h, r, :n], r, seg, k[r])
                is_full = n_valid[h, sel] == TILE
                full[b][h][r] = sel[is_full]
                part[b][h][r] = sel[~is_full]
    return BlockLists(full, part)


# ---------------------------------------------------------------------------------------
# 6. attention
# ---------------------------------------------------------------------------------------

def attention_row_tile(q_rows: np.ndarray, k_tiled: np.ndarray, v_tiled: np.ndarray,
                       keys: np.ndarray, n_valid: np.ndarray, scale: float):
    """Softmax attention of one query tile's rows over the valid slots of the listed key tiles.

    [AGENTS] preamble: attention only visits the selected key tiles. [README]
    Key Features: a single mask function on partial blocks -- reading R12: it
    removes a partial tile's pad slots (slot >= n_valid). Computed directly:
    s = scale q.k over all kept keys, softmax with the row maximum subtracted,
    o = P V / sum(P), lse = log sum exp(s). Rows with no listed key tile give
    o = 0, lse = -inf. q_rows: [R, D]; k_tiled/v_tiled: [nT*128, D] of one head.
    """
    R, D = q_rows.shape
    if len(keys) == 0:
        return np.zeros((R, D)), np.full(R, -np.inf)
    idx = np.concatenate([np.arange(j * TILE, j * TILE + int(n_valid[j])) for j in keys])
    Kk = k_tiled[idx]
    Vk = v_tiled[idx]
    s = scale * (q_rows @ Kk.T)
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    l = p.sum(axis=1, keepdims=True)
    o = (p @ Vk) / l
    lse = (m + np.log(l))[:, 0]
    return o, lse


def attention(q_tiled: np.ndarray, k_tiled: np.ndarray, v_tiled: np.ndarray, n_valid: np.ndarray,
              lists: BlockLists, scale: float, rows: Optional[Sequence[Tuple[int, int, int]]] = None):
    """Block-sparse attention forward over the listed key tiles of every query tile.

    [AGENTS] section 2 (SM90): 128 x 128 tiles at head_dim 128, query tiles of 128
    rows aligned with the key tiles. Reading R13: every slot of a query tile is
    computed, pad slots included (their query is the zero vector from the
    permute), and dropped by the unpermute; softmax scale as given (1/sqrt(128)
    for the workloads here).
    q/k/v_tiled: [B, H, nT*128, D]. ``rows`` optionally restricts the work to some
    (b, h, query tile) triples; other rows are left NaN.
    Returns o [B, H, nT*128, D], lse [B, H, nT*128].
    """
    B, H, Npad, D = q_tiled.shape
    nT = Npad // TILE
    o = np.full((B, H, Npad, D), np.nan)
    lse = np.full((B, H, Npad), np.nan)
    todo = rows if rows is not None else [(b, h, r) for b in range(B) for h in range(H) for r in range(nT)]
    for (b, h, r) in todo:
        keys = np.sort(np.concatenate([lists.full[b][h][r], lists.partial[b][h][r]]))
        sl = slice(r * TILE, (r + 1) * TILE)
        ob, lb = attention_row_tile(q_tiled[b, h, sl], k_tiled[b, h], v_tiled[b, h], keys,
                                    n_valid[h], scale)
        o[b, h, sl] = ob
        lse[b, h, sl] = lb
    return o, lse


def dense_attention_raster(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float,
                           heads: Optional[Sequence[int]] = None):
    """Dense softmax attention in raster order, no tiling: the 100%-density reference.

    Textbook softmax(scale Q K^T) V per (batch, head) over all N tokens.
    q, k, v: [B, N, H, D]. Returns o [B, N, H, D] (NaN on heads not computed), lse [B, N, H].
    """
    B, N, H, D = q.shape
    o = np.full((B, N, H, D), np.nan)
    lse = np.full((B, N, H), np.nan)
    for b in range(B):
        for h in (range(H) if heads is None else heads):
            s = scale * (q[b, :, h, :].astype(np.float64) @ k[b, :, h, :].astype(np.float64).T)
            m = s.max(axis=1, keepdims=True)
            p = np.exp(s - m)
            l = p.sum(axis=1, keepdims=True)
            o[b, :, h, :] = (p @ v[b, :, h, :].astype(np.float64)) / l
            lse[b, :, h] = (m + np.log(l))[:, 0]
    return o, lse


def predictor_param_count(heads: int, blocks: int, D: int = 128) -> int:
    """Parameters of the per-head residual projections (reading R6): 2 * D * 3D per head per block."""
    return 2 * D * 3 * D * heads * blocks


# ---------------------------------------------------------------------------------------
# 7b. attention backward over the same block lists
# ---------------------------------------------------------------------------------------

def transpose_lists(lists: BlockLists, nT_per_head: Sequence[int], nT: int):
    """Query tiles of every key tile: T[b][h][j] = ascending i with j listed for query tile i.

    [README] Key Features / Veda sparse attention: the block-sparse integration carries
    "transposed backward lists" -- the backward walks, for each key tile, the query tiles
    that attended to it. Reading R20: full and partial lists together; key tiles past a
    head's tile count get empty lists.
    """
    B = len(lists.full)
    H = len(lists.full[0])
    out = [[[[] for _ in range(nT)] for _ in range(H)] for _ in range(B)]
    for b in range(B):
        for h in range(H):
            for i in range(int(nT_per_head[h])):
                for j in np.concatenate([lists.full[b][h][i], lists.partial[b][h][i]]):
                    out[b][h][int(j)].append(i)
    return [[[np.array(sorted(t), np.int64) for t in hh] for hh in bb] for bb in out]


def attention_backward(q_tiled: np.ndarray, k_tiled: np.ndarray, v_tiled: np.ndarray, n_valid: np.ndarray,
                       lists: BlockLists, scale: float, o_tiled: np.ndarray, lse: np.ndarray,
                       do_tiled: np.ndarray):
    """Gradients of the block-sparse attention forward with respect to Q, K and V.

    The backward of step 6 for an output gradient dO, over exactly the forward's keys
    (the valid slots of the listed tiles). Per query row q: P = exp(scale q.k - LSE_q),
    D_q = dO_q . O_q, dP = dO_q . v, dS = P (dP - D_q); then dQ_q = scale sum_k dS k,
    dK_k += scale sum_q dS q and dV_k += sum_q P dO_q. Reading R21: pad query slots are
    treated like the forward treats them (computed, with whatever dO they are given); pad
    key slots receive no gradient; rows with no listed key tile give dQ = 0.
    q/k/v/o/do_tiled: [B, H, nT*128, D]; lse: [B, H, nT*128] (the forward's).
    Returns dq, dk, dv [B, H, nT*128, D].
    """
    B, H, Npad, D = q_tiled.shape
    nT = Npad // TILE
    dq = np.zeros((B, H, Npad, D))
    dk = np.zeros((B, H, Npad, D))
    dv = np.zeros((B, H, Npad, D))
    for b in range(B):
        for h in range(H):
            for r in range(nT):
                keys = np.sort(np.concatenate([lists.full[b][h][r], lists.partial[b][h][r]]))
                if len(keys) == 0:
                    continue
                idx = np.concatenate([np.arange(j * TILE, j * TILE + int(n_valid[h, j])) for j in keys])
                sl = slice(r * TILE, (r + 1) * TILE)
                Q, dO, O = q_tiled[b, h, sl], do_tiled[b, h, sl], o_tiled[b, h, sl]
                K, V = k_tiled[b, h, idx], v_tiled[b, h, idx]
                P = np.exp(scale * (Q @ K.T) - lse[b, h, sl][:, None])
                Dq = (dO * O).sum(axis=1, keepdims=True)
                dS = P * (dO @ V.T - Dq)
                dq[b, h, sl] = scale * (dS @ K)
                dk[b, h, idx] += scale * (dS.T @ Q)
                dv[b, h, idx] += P.T @ dO
    return dq, dk, dv


# ---------------------------------------------------------------------------------------
# 8. block heat and mask quality (the predictor's teacher signal and its check)
# ---------------------------------------------------------------------------------------

def block_heat(q_tiled: np.ndarray, k_tiled: np.ndarray, n_valid: np.ndarray,
               nT_per_head: Sequence[int], scale: float,
               rows: Optional[Sequence[Tuple[int, int, int]]] = None) -> np.ndarray:
    """Per-block attention mass of dense attention: the predictor's teacher signal.

    [README] Key Features / Veda sparse attention: the predictor learns from "teacher
    block heat from the dense LSE". Reading R18: heat[b, h, i, j] is the mean, over the
    valid query slots q of tile i, of the sum over the valid key slots k of tile j of
    exp(scale q.k - LSE_q), where LSE_q = log sum_k exp(scale q.k) over every valid key
    of the head (dense attention). A valid row of heat therefore sums to 1 over j. Pad
    query slots do not count; rows past a head's tile count stay 0.
    q/k_tiled: [B, H, nT*128, D]; n_valid: [H, nT]. ``rows`` optionally restricts the
    work to some (b, h, query tile) triples. Returns heat [B, H, nT, nT].
    """
    B, H, Npad, D = q_tiled.shape
    nT = Npad // TILE
    heat = np.zeros((B, H, nT, nT))
    todo = rows if rows is not None else [(b, h, i) for b in range(B) for h in range(H)
                                          for i in range(int(nT_per_head[h]))]
    keys = {}
    for (b, h, i) in todo:
        n = int(nT_per_head[h])
        if (b, h) not in keys:
            idx = np.concatenate([np.arange(j * TILE, j * TILE + int(n_valid[h, j])) for j in range(n)])
            owner = np.concatenate([np.full(int(n_valid[h, j]), j) for j in range(n)])
            keys[(b, h)] = (k_tiled[b, h][idx], owner)
        K, owner = keys[(b, h)]
        nq = int(n_valid[h, i])
        if nq == 0:
            continue
        Q = q_tiled[b, h, i * TILE: i * TILE + nq]
        s = scale * (Q @ K.T)
        m = s.max(axis=1, keepdims=True)
        lse = m + np.log(np.exp(s - m).sum(axis=1, keepdims=True))
        p = np.exp(s - lse)
        heat[b, h, i, :n] = np.bincount(owner, weights=p.sum(axis=0) / nq, minlength=n)
    return heat


def mask_quality(heat: np.ndarray, n_valid: np.ndarray, nT_per_head: Sequence[int],
                 pred: BlockLists, oracle: BlockLists):
    """Attention mass a block mask keeps, and its block recall against the oracle mask.

    [AGENTS] section 4: the predictor is checked by its recall against the oracle mask;
    section 6: at a 10% keep ratio "even an oracle mask" keeps only about 0.63 of the
    attention mass. Reading R19: the oracle mask is the selection step (same budgets,
    forced diagonal, score order) run on heat as the score. The mass a mask keeps in row
    (b, h, i) is the sum of heat[b, h, i, j] over its tiles j; the overall mass is the
    mean over valid query slots (rows weighted by n_valid(i)). Block recall of a row is
    |pred_i & oracle_i| / |oracle_i|; the overall recall is the mean over rows with a
    non-empty oracle list.
    Returns (mass_rows [B, H, nT], recall_rows [B, H, nT], mass, recall).
    """
    B, H, nT, _ = heat.shape
    mass_rows = np.zeros((B, H, nT))
    recall_rows = np.zeros((B, H, nT))
    wsum = msum = 0.0
    rsum, rcount = 0.0, 0
    for b in range(B):
        for h in range(H):
            for i in range(int(nT_per_head[h])):
                mine = set(np.concatenate([pred.full[b][h][i], pred.partial[b][h][i]]).tolist())
                ref = set(np.concatenate([oracle.full[b][h][i], oracle.partial[b][h][i]]).tolist())
                mass_rows[b, h, i] = sum(heat[b, h, i, j] for j in mine)
                w = float(n_valid[h, i])
                wsum += w
                msum += w * mass_rows[b, h, i]
                if ref:
                    recall_rows[b, h, i] = len(mine & ref) / len(ref)
                    rsum += recall_rows[b, h, i]
                    rcount += 1
    return mass_rows, recall_rows, (msum / wsum if wsum else 0.0), (rsum / rcount if rcount else 0.0)


# ---------------------------------------------------------------------------------------
# 9. oracle tile-plan search
# ---------------------------------------------------------------------------------------

def shape_errors(q: np.ndarray, k: np.ndarray, v: np.ndarray, grid: Tuple[int, int, int], n_tail: int,
                 candidates: Sequence[Tuple[int, int, int]], rho: Sequence[Tuple[int, int]],
                 scale: float) -> np.ndarray:
    """Relative output error of every candidate tile shape under its best mask, per head.

    [README] Key Features / Veda sparse attention: "oracle tile-plan search (relative output
    MSE under the best mask)". Reading R22: for head h and shape s, tile the head with s,
    take the oracle mask of section 8 (step 4 on the block heat of s's tiling), run the
    block-sparse attention with it and return sum over valid tokens of |o_s - o_dense|^2
    divided by sum |o_dense|^2, with o_dense the dense attention (section 6's raster
    routine). q, k, v: [B, N, H, D] raster. Returns err [H, len(candidates)] (batch summed).
    """
    B, N, H, D = q.shape
    od, _ = dense_attention_raster(q, k, v, scale)
    err = np.zeros((H, len(candidates)))
    for ci, shape in enumerate(candidates):
        m = tile_map(grid, tuple(shape), n_tail)
        slots, n_valid, segment = stack_maps([m] * H)
        nT_h = [len(m.n_valid)] * H
        qt, kt, vt = permute(q, slots), permute(k, slots), permute(v, slots)
        heat = block_heat(qt, kt, n_valid, nT_h, scale)
        mask = select(heat, n_valid, segment, nT_h, rho)
        o_t, _ = attention(qt, kt, vt, n_valid, mask, scale)
        o = unpermute(np.nan_to_num(o_t), slots, N)
        for h in range(H):
            num = ((o[:, :, h] - od[:, :, h]) ** 2).sum()
            den = (od[:, :, h] ** 2).sum()
            err[h, ci] = num / den
    return err


def tile_plan(err: np.ndarray, max_shapes: int = 2) -> Tuple[List[int], np.ndarray]:
    """Majority vote over the heads' best shapes, at most `max_shapes` shapes per layer.

    [README] Key Features: "majority vote, at most two shapes per layer". Reading R22: each
    head votes for its lowest-error candidate (ties to the earlier candidate); the layer
    keeps the `max_shapes` candidates with the most votes (ties to the earlier candidate);
    every head then takes whichever kept candidate has its lower error (ties to the earlier).
    err: [H, C]. Returns (kept candidate indices, per-head candidate index [H]).
    """
    H, C = err.shape
    votes = np.bincount(np.argmin(err, axis=1), minlength=C)
    order = sorted(range(C), key=lambda c: (-votes[c], c))
    kept = [c for c in order[:max_shapes] if votes[c] > 0] or [order[0]]
    kept = sorted(kept)
    assign = np.array([kept[int(np.argmin(err[h, kept]))] for h in range(H)])
    return kept, assign


# ---------------------------------------------------------------------------------------
# 10. FP8 (e4m3) variant of the attention step
# ---------------------------------------------------------------------------------------
# The pages ship their predictor in FP8 ([AGENTS] preamble and section 3) but give no FP8
# attention; the variant here is defined by this module. Reading R23: Q, K and V tiles are quantised
# to e4m3 (OCP FP8 E4M3 "fn": 1 sign, 4 exponent bits with bias 7, 3 mantissa bits, no
# infinities, codes 0x7F / 0xFF are NaN) with one scale per (batch, head) tensor:
# scale = amax / 448 and code = e4m3(x * (448 / amax)), both in fp32, rounding to nearest
# even and saturating to +-448; an all-zero tensor gets scale 1. V is stored as transposed
# tiles (each 128 x 128 tile as [head-dim channel][key slot]). The attention of the FP8
# variant is then the attention step on the dequantised tensors (code value * scale).

E4M3_MAX = 448.0


def e4m3_round(x: np.ndarray) -> np.ndarray:
    """Nearest e4m3 value of every element of x (float64 in, float64 out), ties to even,
    saturating at +-448 (R23). The quantum of x's binade is 2^(floor(log2 |x|) - 3) for
    normals (|x| >= 2^-6) and 2^-9 for subnormals; 448 = 1.75 * 2^8 is the largest finite."""
    x = np.asarray(x, dtype=np.float64)
    if not np.all(np.isfinite(x)):
        raise ValueError("e4m3_round: non-finite input")
    a = np.abs(x)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.clip(e, -6, 8)
    quantum = np.ldexp(1.0, (e - 3).astype(np.int64))
    v = np.minimum(np.round(a / quantum) * quantum, E4M3_MAX)   # np.round: half to even
    return np.copysign(v, x)


def e4m3_codes(x: np.ndarray) -> np.ndarray:
    """uint8 e4m3 codes of the nearest e4m3 values of x (see e4m3_round); -0 keeps its sign bit."""
    x = np.asarray(x, dtype=np.float64)
    v = np.abs(e4m3_round(x))
    codes = np.zeros(x.shape, dtype=np.uint8)
    sub = (v > 0) & (v < 2.0 ** -6)
    codes[sub] = np.round(v[sub] / 2.0 ** -9).astype(np.uint8)          # exponent field 0
    nrm = v >= 2.0 ** -6
    E = np.floor(np.log2(v[nrm]))
    mant = np.round(v[nrm] / np.ldexp(1.0, E.astype(np.int64)) * 8 - 8).astype(np.int64)
    codes[nrm] = (((E.astype(np.int64) + 7) << 3) | mant).astype(np.uint8)
    codes[np.signbit(x)] |= np.uint8(0x80)
    return codes


def e4m3_value(codes: np.ndarray) -> np.ndarray:
    """float64 value of e4m3 codes (NaN codes 0x7F / 0xFF are rejected)."""
    c = np.asarray(codes, dtype=np.int64)
    if np.any((c & 0x7F) == 0x7F):
        raise ValueError("e4m3_value: NaN code")
    ef, m = (c >> 3) & 0xF, c & 7
    mag = np.where(ef == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.ldexp(1.0, ef - 7))
    return np.where(c & 0x80, -mag, mag)


def quantize_fp8(x_tiled: np.ndarray, transpose_tiles: bool = False):
    """Per-(batch, head) e4m3 quantisation of tiled tensors [B, H, nT*128, D] (R23).
    Returns (codes uint8 [B, H, nT*128, D], scale float32 [B, H]); with transpose_tiles every
    128 x D tile of the codes is stored transposed (D = 128)."""
    B, H, Npad, D = x_tiled.shape
    x32 = x_tiled.astype(np.float32)
    amax = np.abs(x32).max(axis=(2, 3)).astype(np.float32)
    safe = np.where(amax > 0, amax, np.float32(E4M3_MAX)).astype(np.float32)
    inv = (np.float32(E4M3_MAX) / safe).astype(np.float32)               # 1 for a zero tensor
    scale = (safe / np.float32(E4M3_MAX)).astype(np.float32)
    y = (x32 * inv[:, :, None, None]).astype(np.float32)
    codes = e4m3_codes(y.astype(np.float64))
    if transpose_tiles:
        codes = codes.reshape(B, H, Npad // TILE, TILE, D).swapaxes(3, 4).reshape(B, H, Npad, D)
    return codes, scale


def dequantize_fp8(codes: np.ndarray, scale: np.ndarray, transposed_tiles: bool = False) -> np.ndarray:
    """float64 tensor [B, H, nT*128, D] of quantize_fp8's output (code value * scale)."""
    B, H, Npad, D = codes.shape
    c = codes
    if transposed_tiles:
        c = c.reshape(B, H, Npad // TILE, D, TILE).swapaxes(3, 4).reshape(B, H, Npad, D)
    return e4m3_value(c) * scale.astype(np.float64)[:, :, None, None]


# ---------------------------------------------------------------------------------------
# whole path
# ---------------------------------------------------------------------------------------

def run_path(q, k, v, Wq, Wk, grid, head_shapes, n_tail, rho, scale, tile_orders=None):
    """All steps in order on raster inputs [B, N, H, D] (float64). Returns a dict of every stage."""
    H = q.shape[2]
    maps = [tile_map(grid, tuple(head_shapes[h]), n_tail,
                     None if tile_orders is None else tile_orders[h]) for h in range(H)]
    nT_per_head = [len(m.n_valid) for m in maps]
    slots, n_valid, segment = stack_maps(maps)
    qt, kt, vt = permute(q, slots), permute(k, slots), permute(v, slots)
    pq, pk = pool(qt, n_valid), pool(kt, n_valid)
    S = scores(pq, pk, Wq, Wk)
    lists = select(S, n_valid, segment, nT_per_head, rho)
    o_t, lse = attention(qt, kt, vt, n_valid, lists, scale)
    o = unpermute(np.nan_to_num(o_t), slots, q.shape[1])
    return dict(slots=slots, n_valid=n_valid, segment=segment, nT_per_head=nT_per_head,
                q_tiled=qt, k_tiled=kt, v_tiled=vt, pooled_q=pq, pooled_k=pk, scores=S,
                lists=lists, o_tiled=o_t, lse=lse, o=o)
