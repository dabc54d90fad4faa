"""Shared machinery of the GPU parity tests: run the oracle and the CUDA library on the
same seeded inputs, stage by stage, and compare them with the stated tolerances.

Tolerances (fixed by the method's parity rule):
  * tile maps, permute, unpermute, block lists: bit-exact (lists: the oracle's selection
    is fed the GPU's fp32 scores);
  * scores: |gpu - ref| <= 1e-3 * max(|ref|, mean |ref| over the head's matrix);
  * attention output (bf16-rounded inputs, identical lists): max abs error <= 2e-2 and
    mean abs error <= 2e-3 against fp64;
  * pooling (not fixed by the rule): max/min exact, mean within 1e-5 relative (fp32 sum).
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np
import torch

import synth
from oracle import veda_oracle as O

SCORE_RTOL = 1e-3
ATTN_MAX_ABS = 2e-2
ATTN_MEAN_ABS = 2e-3
SCALE = 1.0 / math.sqrt(128)


def veda():
    from block_sparse_attention_max_b200 import veda as V
    return V


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().double().numpy()


def oracle_maps(w: synth.Workload, orders: Optional[np.ndarray]):
    cache = {}
    maps = []
    for h in range(w.H):
        key = (tuple(w.head_shapes[h]), None if orders is None else orders[h].tobytes())
        if key not in cache:
            cache[key] = O.tile_map(w.grid, w.head_shapes[h], w.n_tail,
                                    None if orders is None else orders[h])
        maps.append(cache[key])
    slots, nv, seg = O.stack_maps(maps, w.nT)
    return slots, nv, seg, [len(m.n_valid) for m in maps]


def lists_to_device(lists: O.BlockLists, B: int, H: int, nT: int, stride: int, device):
    V = veda()
    fc = np.zeros((B, H, nT), np.int32)
    pc = np.zeros((B, H, nT), np.int32)
    fi = np.zeros((B, H, nT, stride), np.int32)
    pi = np.zeros((B, H, nT, stride), np.int32)
    for b in range(B):
        for h in range(H):
            for r in range(nT):
                f, p = lists.full[b][h][r], lists.partial[b][h][r]
                fc[b, h, r], pc[b, h, r] = len(f), len(p)
                fi[b, h, r, :len(f)] = f
                pi[b, h, r, :len(p)] = p
    t = lambda a: torch.from_numpy(a).to(device)
    return V.BlockLists(t(fc), t(fi), t(pc), t(pi), stride)


def gpu_lists_equal(gl, lists: O.BlockLists, heads: Sequence[int], rows=None) -> Tuple[int, int]:
    """Compare the GPU lists of some heads with oracle lists (oracle head index = position)."""
    fc, fi = gl.full_cnt.cpu().numpy(), gl.full_idx.cpu().numpy()
    pc, pi = gl.part_cnt.cpu().numpy(), gl.part_idx.cpu().numpy()
    bad = total = 0
    B = fc.shape[0]
    for b in range(B):
        for j, h in enumerate(heads):
            for r in (range(fc.shape[2]) if rows is None else rows):
                total += 1
                f, p = lists.full[b][j][r], lists.partial[b][j][r]
                ok = (fc[b, h, r] == len(f) and pc[b, h, r] == len(p)
                      and (fi[b, h, r, :len(f)] == f).all() and (pi[b, h, r, :len(p)] == p).all())
                bad += not ok
    return bad, total


def fp8_v_key_positions() -> np.ndarray:
    """Key slot at each key position of a transposed V tile of veda_quantize_fp8: within every
    group of 16, position 4c + e holds slot 2c + (e % 2) + 8 (e // 2) (include/veda.h)."""
    pos = np.arange(128)
    m, c, e = pos // 16, (pos % 16) // 4, pos % 4
    return 16 * m + 2 * c + (e % 2) + 8 * (e // 2)


def fp8_v_layout(codes_t: np.ndarray) -> np.ndarray:
    """Oracle codes with plainly transposed tiles ([..., channel, key slot]) in the library's
    key order."""
    return codes_t[..., fp8_v_key_positions()]


def score_errors(gpu: np.ndarray, ref: np.ndarray) -> float:
    """Worst |gpu - ref| / max(|ref|, mean|ref| of the head's matrix) over all entries."""
    worst = 0.0
    for idx in np.ndindex(*ref.shape[:2]):
        r = ref[idx]
        g = gpu[idx]
        floor = np.abs(r).mean()
        worst = max(worst, float((np.abs(g - r) / np.maximum(np.abs(r), floor)).max()))
    return worst


def attn_errors(gpu: np.ndarray, ref: np.ndarray) -> Tuple[float, float]:
    d = np.abs(gpu - ref)
    return float(d.max()), float(d.mean())
