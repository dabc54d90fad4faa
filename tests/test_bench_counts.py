"""bench.py's work and traffic counts, on hand-built block lists (CPU only).

The bench line's FLOP figures come from these helpers: visited blocks (4 * 128^3 FLOP each,
the rate the target is stated on), the FLOP the forward kernel issues (a key tile with at
most 64 valid slots is computed over its first 64 keys) and the FLOP over valid query x
valid key pairs. Each is checked here against a brute-force count over the same lists.
"""
import dataclasses
import hashlib
import json
import os

import numpy as np
import torch

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@dataclasses.dataclass
class _Lists:
    full_cnt: torch.Tensor
    full_idx: torch.Tensor
    part_cnt: torch.Tensor
    part_idx: torch.Tensor


def _lists(rows, nT, stride):
    """rows[b][h][r] = (full key tiles, partial key tiles); -1 pads the unused entries."""
    B, H = len(rows), len(rows[0])
    fc = torch.zeros((B, H, nT), dtype=torch.int32)
    pc = torch.zeros((B, H, nT), dtype=torch.int32)
    fi = torch.full((B, H, nT, stride), -1, dtype=torch.int32)
    pi = torch.full((B, H, nT, stride), -1, dtype=torch.int32)
    for b in range(B):
        for h in range(H):
            for r in range(nT):
                f, p = rows[b][h][r]
                fc[b, h, r], pc[b, h, r] = len(f), len(p)
                fi[b, h, r, :len(f)] = torch.tensor(f, dtype=torch.int32)
                pi[b, h, r, :len(p)] = torch.tensor(p, dtype=torch.int32)
    return _Lists(fc, fi, pc, pi)


def _case():
    # two heads, four tiles each; valid slots per tile differ by head
    tile_valid = np.array([[128, 36, 128, 96], [128, 64, 65, 1]], dtype=np.int32)
    rows = [[
        [([0, 2], [1]), ([0], [1, 3]), ([2], []), ([0, 2], [3])],           # head 0
        [([0], [1, 2, 3]), ([0], [1]), ([], [2]), ([0], [3])],              # head 1
    ]]
    return _lists(rows, 4, 4), tile_valid, rows


def test_visited_blocks_count_every_list_entry():
    lists, _, rows = _case()
    want = sum(len(f) + len(p) for bb in rows for hh in bb for (f, p) in hh)
    assert bench._visited_blocks(lists) == want == 19


def test_executed_flop_halves_partial_tiles_of_at_most_64_slots():
    lists, tv, rows = _case()
    half = 0
    for h, hh in enumerate(rows[0]):
        for (_, p) in hh:
            half += sum(1 for j in p if tv[h][j] <= 64)
    assert half == 6   # head 0: tile 1 (36 slots) twice; head 1: tile 1 (64) twice, tile 3 (1) twice
    want = (19 - half) * bench.FLOP_PER_BLOCK + half * bench.FLOP_PER_BLOCK / 2
    assert bench._executed_flop(lists, tv) == want


def test_valid_token_flop_counts_valid_query_times_valid_key_pairs():
    lists, tv, rows = _case()
    pairs = 0
    for h, hh in enumerate(rows[0]):
        for r, (f, p) in enumerate(hh):
            pairs += int(tv[h][r]) * sum(int(tv[h][j]) for j in list(f) + list(p))
    assert bench._valid_token_flop(lists, tv) == 4.0 * 128 * pairs


def test_traffic_record_is_used_only_for_its_kernel_source_and_scales_with_heads():
    rec = json.load(open(os.path.join(ROOT, "profiles", "attn_fwd_clip16x9.traffic.json")))
    src = os.path.join(ROOT, rec["kernel_source"])
    assert rec["dram_bytes_per_launch"] == rec["dram_bytes_read"] + rec["dram_bytes_write"]
    if rec["kernel_source_sha256"] != hashlib.sha256(open(src, "rb").read()).hexdigest():
        # counters of another version of the kernel: the bench line reports no traffic
        assert bench._attn_traffic(rec["heads"]) is None
        return
    assert bench._attn_traffic(rec["heads"]) == rec["dram_bytes_per_launch"]
    assert bench._attn_traffic(5 * rec["heads"]) == 5 * rec["dram_bytes_per_launch"]
