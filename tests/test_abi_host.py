"""The C-ABI library without a GPU: it loads, exports every symbol include/veda.h
declares, its host-side tile maps match the oracle's bit for bit, and device calls
validate their arguments before touching CUDA (and never fall back to anything)."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import synth
from oracle import veda_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
veda = pytest.importorskip("block_sparse_attention_max_b200.veda")


@pytest.fixture(scope="module")
def L():
    from block_sparse_attention_max_b200 import build
    build.build()
    return veda.lib()


def _declared():
    src = open(os.path.join(ROOT, "include", "veda.h")).read()
    return sorted(set(re.findall(r"VEDA_API\s+[\w\s\*]+?\b(veda_\w+)\s*\(", src)))


def test_exports_every_declared_symbol(L):
    names = _declared()
    assert len(names) >= 13
    assert sorted(veda.EXPORTED) == names
    for n in names:
        assert hasattr(L, n), n
    assert L.veda_abi_version() == 1
    assert L.veda_status_string(0) == b"ok"


@pytest.mark.parametrize("w", [synth.TINY, synth.SMALL, synth.CLIP16x9, synth.MIXED])
def test_tile_map_matches_oracle(L, w):
    inp_order = synth.tile_orders(w)
    maps = veda.build_tile_map(w.grid, w.head_shapes, w.n_tail, inp_order)
    assert (maps.N, maps.nT, maps.Npad) == (w.N, w.nT, w.Npad)
    om = [O.tile_map(w.grid, w.head_shapes[h], w.n_tail, None if inp_order is None else inp_order[h])
          for h in range(w.H)]
    slots, nv, seg = O.stack_maps(om, w.nT)
    assert (maps.tile_map == slots).all()
    assert (maps.tile_valid == nv).all()
    assert (maps.tile_segment == seg).all()
    assert (maps.nT_per_head == [len(m.n_valid) for m in om]).all()


def test_tile_map_ragged_heads_and_rejections(L):
    shapes = [(1, 8, 16), (2, 8, 8), (4, 4, 8)]
    maps = veda.build_tile_map((5, 8, 16), shapes, 0)
    assert list(maps.nT_per_head) == [5, 6, 8] and maps.nT == 8
    om = [O.tile_map((5, 8, 16), s) for s in shapes]
    slots, nv, seg = O.stack_maps(om, 8)
    assert (maps.tile_map == slots).all() and (maps.tile_valid == nv).all()
    with pytest.raises(veda.VedaError):
        veda.build_tile_map((4, 8, 16), [(2, 8, 16)], 0)          # not 128 tokens
    with pytest.raises(veda.VedaError):
        veda.build_tile_map((4, 8, 16), [(1, 8, 16)], 0, np.zeros((1, 4), np.int32))  # not a permutation


def test_device_calls_validate_before_cuda(L):
    INVALID, UNSUPPORTED = 1, 2
    assert L.veda_permute_tiles(None, None, None, 1, 1, 1, 128, 128, None) == INVALID
    assert L.veda_permute_tiles(16, 16, 16, 1, 1, 1, 64, 128, None) == UNSUPPORTED
    assert L.veda_permute_tiles(16, 16, 16, 1, 1, 1, 128, 100, None) == INVALID
    assert L.veda_tile_pool(None, None, None, 1, 1, 1, 128, None) == INVALID
    assert L.veda_block_scores(16, 16, 16, 16, 16, 256, 0, 1, 1, 4, 128, None) == INVALID  # workspace too small
    num = (ctypes.c_int32 * 1)(1)
    den = (ctypes.c_int32 * 1)(0)
    assert L.veda_select_blocks(16, 16, 16, 16, 1, ctypes.addressof(num), ctypes.addressof(den),
                                16, 16, 16, 16, 4, 1, 1, 4, None) == INVALID          # den = 0
    den[0] = 2
    assert L.veda_select_blocks(16, 16, 16, 16, 1, ctypes.addressof(num), ctypes.addressof(den),
                                16, 16, 16, 16, 1, 1, 1, 8, None) == INVALID          # stride too small
    assert L.veda_select_blocks(16, 16, 16, 16, 1, ctypes.addressof(num), ctypes.addressof(den),
                                16, 16, 16, 16, 2049, 1, 1, 2049, None) == INVALID    # nT above VEDA_MAX_TILES
    num5 = (ctypes.c_int32 * 5)(1, 1, 1, 1, 1)
    den5 = (ctypes.c_int32 * 5)(2, 2, 2, 2, 2)
    assert L.veda_select_blocks(16, 16, 16, 16, 5, ctypes.addressof(num5), ctypes.addressof(den5),
                                16, 16, 16, 16, 8, 1, 1, 8, None) == INVALID          # five segments
    assert L.veda_block_sparse_attn_fwd(16, 16, 16, 16, 16, 16, 16, 16, 4, -1.0, 16, None,
                                        1, 1, 4, 128, None) == INVALID                 # bad scale
    assert L.veda_block_sparse_attn_fwd(8, 16, 16, 16, 16, 16, 16, 16, 4, 0.1, 16, None,
                                        1, 1, 4, 128, None) == INVALID                 # misaligned q
    assert L.veda_block_heat(16, 16, 16, 16, 16, 16, 16, 4, None, 0.1, 16,
                             1, 1, 4, 128, None) == INVALID                            # no LSE
    assert L.veda_block_heat(16, 16, 16, 16, 16, 16, 16, 4, 16, 0.1, 16,
                             1, 1, 4, 64, None) == UNSUPPORTED                         # head_dim 64
    assert L.veda_block_heat(16, 24, 16, 16, 16, 16, 16, 4, 16, 0.1, 16,
                             1, 1, 4, 128, None) == INVALID                            # misaligned k
    args = [16] * 7 + [4] + [16] * 4 + [4] + [16] * 3
    assert L.veda_mask_quality(*args, 1, 1, 4096, None) == INVALID                     # nT too large
    assert L.veda_mask_quality(*args[:-1], None, 1, 1, 4, None) == INVALID             # no totals
    # FP8 variant
    assert L.veda_quantize_fp8(None, 16, 16, 1, 1, 4, 128, 0, None) == INVALID          # no input
    assert L.veda_quantize_fp8(16, 16, 16, 1, 1, 4, 128, 2, None) == INVALID            # transpose 2
    assert L.veda_quantize_fp8(16, 16, 16, 1, 1, 4, 64, 0, None) == UNSUPPORTED         # head_dim 64
    assert L.veda_quantize_fp8(16, 24, 16, 1, 1, 4, 128, 0, None) == INVALID            # misaligned codes
    f8 = [16] * 11
    assert L.veda_block_sparse_attn_fwd_fp8(*([None] + f8[1:]), 4, 0.1, 16, 16, 1, 1, 4, 128, None) == INVALID
    assert L.veda_block_sparse_attn_fwd_fp8(*f8, 4, -1.0, 16, 16, 1, 1, 4, 128, None) == INVALID   # bad scale
    assert L.veda_block_sparse_attn_fwd_fp8(*f8, 4, 0.1, 16, 16, 1, 1, 4, 64, None) == UNSUPPORTED
    assert L.veda_block_sparse_attn_fwd_fp8(*([24] + f8[1:]), 4, 0.1, 16, 16, 1, 1, 4, 128, None) == INVALID
    assert veda.block_scores_workspace_bytes(1, 2, 4) == 2 * 2 * 4 * 128 * 4


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU behaviour")
def test_no_device_means_error_not_fallback(L):
    # well-formed arguments reach the device query, which fails without a GPU
    st = L.veda_permute_tiles(256, 256, 256, 1, 128, 1, 128, 128, None)
    assert st in (2, 3)
    assert L.veda_check_device_status(None, None) == 3


def test_tile_plan_vote_hand_examples(L):
    # the oracle's hand-worked votes, through the C ABI
    err = np.array([[0.1, 0.2, 0.3],
                    [0.5, 0.4, 0.3],
                    [0.9, 0.8, 0.1],
                    [0.3, 0.1, 0.4],
                    [0.6, 0.6, 0.5]])
    kept, assign = veda.tile_plan_vote(err)
    assert kept == [0, 2] and assign.tolist() == [0, 2, 2, 0, 2]
    kept, assign = veda.tile_plan_vote(err, max_shapes=1)
    assert kept == [2] and assign.tolist() == [2] * 5
    kept, assign = veda.tile_plan_vote(err, max_shapes=3)
    assert kept == [0, 1, 2] and assign.tolist() == [0, 2, 2, 1, 2]
    kept, assign = veda.tile_plan_vote(np.array([[0.1, 0.2], [0.2, 0.3]]))
    assert kept == [0] and assign.tolist() == [0, 0]
    kept, assign = veda.tile_plan_vote(np.array([[0.2, 0.2, 0.2]]), max_shapes=1)
    assert kept == [0] and assign.tolist() == [0]


def test_tile_plan_vote_matches_oracle_on_random_matrices(L):
    # errors on a coarse grid, so that equal errors and equal vote counts are common
    rng = np.random.default_rng(123)
    for _ in range(300):
        H, C = int(rng.integers(1, 12)), int(rng.integers(1, 7))
        err = rng.integers(0, 5, size=(H, C)) / 4.0
        for ms in (1, 2, 3):
            kept, assign = veda.tile_plan_vote(err, ms)
            kept_o, assign_o = O.tile_plan(err, ms)
            assert kept == list(kept_o) and assign.tolist() == assign_o.tolist(), (err, ms)


def test_tile_plan_vote_rejects_nan_and_bad_sizes(L):
    with pytest.raises(veda.VedaError):
        veda.tile_plan_vote(np.array([[0.1, np.nan]]))
    with pytest.raises(veda.VedaError):
        veda.tile_plan_vote(np.zeros((2, 3)), max_shapes=0)


def test_binding_checks_shapes_before_passing_pointers():
    """A buffer of the wrong shape would send a kernel outside it: the binding compares every
    tensor's shape with the call's sizes (and the tile map's and the lists') before the call."""
    maps = veda.build_tile_map((2, 8, 16), [(1, 8, 16), (1, 8, 16)], 0).to("cpu")   # H = 2, nT = 2
    veda._need_maps(maps, 2, 256, cuda=False)
    with pytest.raises(ValueError, match="slots per head"):
        veda._need_maps(maps, 2, 384, cuda=False)
    with pytest.raises(ValueError, match="expected shape"):
        veda._need_maps(maps, 3, 256, cuda=False)                  # three heads, map of two
    z = lambda *s: torch.zeros(s, dtype=torch.int32)
    lists = veda.BlockLists(z(1, 2, 2), z(1, 2, 2, 2), z(1, 2, 2), z(1, 2, 2, 2), 2)
    veda._need_lists(lists, 1, 2, 2, cuda=False)
    with pytest.raises(ValueError, match="stride"):
        veda._need_lists(veda.BlockLists(z(1, 2, 2), z(1, 2, 2, 3), z(1, 2, 2), z(1, 2, 2, 3), 3), 1, 2, 2,
                         cuda=False)
    with pytest.raises(ValueError, match="expected shape"):
        veda._need_lists(lists, 2, 2, 2, cuda=False)                # batch 2, lists of batch 1
    with pytest.raises(ValueError, match="expected shape"):
        veda._need_lists(veda.BlockLists(z(1, 2, 2), z(1, 2, 2, 1), z(1, 2, 2), z(1, 2, 2, 2), 2), 1, 2, 2,
                         cuda=False)                                 # full_idx narrower than the stride
    with pytest.raises(TypeError):
        veda._need(torch.zeros(4, dtype=torch.float16), torch.bfloat16, "x", cuda=False)
    with pytest.raises(ValueError, match="expected shape"):
        veda._need(torch.zeros(4, 3, dtype=torch.bfloat16), torch.bfloat16, "x", cuda=False, shape=(4, 4))
    veda._need(torch.zeros(4, 4, dtype=torch.bfloat16), torch.bfloat16, "x", cuda=False, shape=(4, 4))
