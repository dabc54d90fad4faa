"""GPU parity of the teacher block heat and of the mask-quality step, through the C ABI.

Heat: the GPU runs its own chain -- permute, every key tile listed (selection at density
1/1), dense attention for the LSE, block heat -- and is compared with the oracle's heat,
computed in fp64 from the same bf16 tiles with its own dense LSE. Tolerance (derived from
the arithmetic): the GPU's scores are fp32 sums of bf16 products (~1e-6 relative to |s|,
and |scale * s| stays below ~15 here), its LSE comes from the same scores, ex2.approx is
within ~2^-22 relative and the block sums are fp32, so |gpu - ref| <= 2e-4 |ref| + 1e-7.
Mask quality: both sides select the oracle mask on the GPU's heat (bit-exact lists, as for
the predicted scores), and the kept mass and recall of the pipeline's predicted mask are
compared with the oracle's mask_quality on that heat: per row within 1e-5 relative (fp32
sums over one row's blocks); the job totals are fp32 atomic sums of one term per row in
whatever order the rows finish, so within n_rows * 2^-24 relative (the worst case of n
fp32 additions), at least 1e-5.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import veda_oracle as O
import parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
HEAT_RTOL, HEAT_ATOL = 2e-4, 1e-7


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from block_sparse_attention_max_b200 import build
    build.build()
    V = P.veda()
    V.lib()
    yield
    V.check_device_status()


def _oracle_lists(gl, heads):
    """GPU block lists of some heads as the oracle's BlockLists."""
    fc, fi = gl.full_cnt.cpu().numpy(), gl.full_idx.cpu().numpy()
    pc, pi = gl.part_cnt.cpu().numpy(), gl.part_idx.cpu().numpy()
    B, _, nT = fc.shape
    full = [[[fi[b, h, r, :fc[b, h, r]].astype(np.int64) for r in range(nT)] for h in heads] for b in range(B)]
    part = [[[pi[b, h, r, :pc[b, h, r]].astype(np.int64) for r in range(nT)] for h in heads] for b in range(B)]
    return O.BlockLists(full, part)


def _run(w, heads=None, rows=None, check_quality=True):
    V = P.veda()
    inp = synth.make_inputs(w)
    orders = inp.tile_order
    slots, nv, seg, nTh = P.oracle_maps(w, orders)
    maps = V.build_tile_map(w.grid, w.head_shapes, w.n_tail, orders).to(DEV)
    q_d, k_d, v_d, wq, wk = (t.to(DEV) for t in (inp.q, inp.k, inp.v, inp.wq, inp.wk))
    bufs = V.sparse_attention(q_d, k_d, v_d, wq, wk, maps, w.rho, P.SCALE)   # the predicted mask
    qt, kt, vt = bufs.q_t, bufs.k_t, bufs.v_t
    B, H, Npad, D = qt.shape
    nT = Npad // 128
    dense = V.select_blocks(torch.zeros((B, H, nT, nT), dtype=torch.float32, device=DEV), maps,
                            [(1, 1)] * len(w.rho))
    _, lse = V.block_sparse_attn_fwd(qt, kt, vt, maps, dense, P.SCALE)
    heat = V.block_heat(qt, kt, maps, dense, lse, P.SCALE)
    V.check_device_status()
    heat_g = P.f64(heat)

    # every valid row of the GPU's heat sums to 1; rows past a head's tiles are 0
    for h in range(H):
        n = nTh[h]
        sums = heat_g[:, h, :n, :n].sum(axis=-1)
        assert np.allclose(sums, 1.0, atol=1e-4), f"head {h}: heat rows sum to {sums.min()}..{sums.max()}"
        assert not heat_g[:, h, n:].any()

    # heat against the oracle on the checked heads / rows
    hs = list(range(H)) if heads is None else list(heads)
    oq = O.permute(P.f64(inp.q[:, :, hs]), slots[hs])
    ok_ = O.permute(P.f64(inp.k[:, :, hs]), slots[hs])
    todo = [(b, j, i) for b in range(B) for j, h in enumerate(hs)
            for i in (range(nTh[h]) if rows is None else [r for r in rows if r < nTh[h]])]
    heat_o = O.block_heat(oq, ok_, nv[hs], [nTh[h] for h in hs], P.SCALE, rows=todo)
    for (b, j, i) in todo:
        g, r = heat_g[b, hs[j], i], heat_o[b, j, i]
        assert np.all(np.abs(g - r) <= HEAT_RTOL * np.abs(r) + HEAT_ATOL), \
            f"heat differs at b{b} h{hs[j]} i{i}: max abs {np.abs(g - r).max():.3g}"

    if not check_quality:
        return heat
    # the oracle mask selected on the GPU's heat, by both sides
    orc = V.select_blocks(heat, maps, w.rho)
    orc_o = O.select(heat_g, nv, seg, nTh, w.rho)
    bad, total = P.gpu_lists_equal(orc, orc_o, list(range(H)))
    assert bad == 0, f"{bad} of {total} oracle-mask rows differ"
    q_g = V.mask_quality(heat, maps, bufs.lists, orc)
    V.check_device_status()
    pred_o = _oracle_lists(bufs.lists, list(range(H)))
    mass_rows, recall_rows, mass, recall = O.mask_quality(heat_g, nv, nTh, pred_o, orc_o)
    assert np.allclose(P.f64(q_g.mass_rows), mass_rows, rtol=1e-5, atol=1e-7)
    assert np.allclose(P.f64(q_g.recall_rows), recall_rows, rtol=0, atol=1e-6)
    n_rows = B * sum(nTh[h] for h in range(H))            # one total term per query tile
    tot_rel = max(1e-5, n_rows * 2.0 ** -24)
    assert q_g.mass == pytest.approx(mass, rel=tot_rel)
    assert q_g.recall == pytest.approx(recall, rel=tot_rel)
    # the oracle mask keeps at least the predicted mask's mass in every row
    q_or = V.mask_quality(heat, maps, orc, orc)
    assert q_or.recall == pytest.approx(1.0)
    assert np.all(P.f64(q_or.mass_rows) >= P.f64(q_g.mass_rows) - 1e-5)
    return heat


def test_heat_tiny():
    _run(synth.TINY)


def test_heat_small():
    _run(synth.SMALL, heads=[0, 5])


def test_heat_mixed_shapes_tail_and_segments():
    _run(synth.MIXED, heads=[0, 17, 31], rows=[0, 1, 100, 223, 224, 228])


def test_heat_clip16x9_sampled():
    _run(synth.CLIP16x9, heads=[0, 39], rows=[0, 247, 495], check_quality=False)


def test_heat_ragged_heads_batch_and_empty_rows():
    w = synth.Workload("ragged", 9, B=2, H=3, grid=(5, 8, 16),
                       head_shapes=((1, 8, 16), (2, 8, 8), (4, 4, 8)), n_tail=0,
                       rho=((1, 2),), field="smooth")
    _run(w)
