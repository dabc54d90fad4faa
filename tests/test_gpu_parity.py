"""GPU parity: every step of the CUDA library against the fp64 oracle, through the C ABI.

Stage tests feed both sides the same seeded inputs (the oracle's own output of the
previous step, never the GPU's -- except the block selection, which the parity rule
feeds the GPU's fp32 scores). The end-to-end tests run the public ``sparse_attention``
path and compare every intermediate. Full-size workloads compare sampled heads and
query tiles, in the launch configuration the benchmark times.
"""
import math

import numpy as np
import pytest
import torch

import synth
from oracle import veda_oracle as O
import parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from block_sparse_attention_max_b200 import build
    build.build()
    V = P.veda()
    V.lib()
    yield
    V.check_device_status()


def _stage_run(w: synth.Workload, heads=None, rows=None, attn_rows=None):
    """Stage-by-stage parity on workload w. heads: oracle heads checked (all if None)."""
    V = P.veda()
    inp = synth.make_inputs(w)
    orders = inp.tile_order
    slots, nv, seg, nTh = P.oracle_maps(w, orders)
    hm = V.build_tile_map(w.grid, w.head_shapes, w.n_tail, orders)
    assert (hm.tile_map == slots).all() and (hm.tile_valid == nv).all()
    maps = hm.to(DEV)
    hs = list(range(w.H)) if heads is None else list(heads)

    # 1. permute: bit-exact
    q_d, k_d, v_d = (t.to(DEV) for t in (inp.q, inp.k, inp.v))
    qt = V.permute_tiles(q_d, maps)
    kt = V.permute_tiles(k_d, maps)
    vt = V.permute_tiles(v_d, maps)
    V.check_device_status()
    xq = P.f64(inp.q[:, :, hs])
    oq = O.permute(xq, slots[hs])
    assert np.array_equal(P.f64(qt[:, hs]), oq), "permute differs"
    ok_ = O.permute(P.f64(inp.k[:, :, hs]), slots[hs])
    ov_ = O.permute(P.f64(inp.v[:, :, hs]), slots[hs])

    # 2. pool (input: the oracle's tiles, as bf16 -- the same bytes)
    pq_g = V.tile_pool(qt, maps)
    pk_g = V.tile_pool(kt, maps)
    pq_o = O.pool(oq, nv[hs])
    pk_o = O.pool(ok_, nv[hs])
    for g_, o_ in ((P.f64(pq_g[:, hs]), pq_o), (P.f64(pk_g[:, hs]), pk_o)):
        assert np.array_equal(g_[..., 1:, :], o_[..., 1:, :]), "max/min differ"
        assert np.allclose(g_[..., 0, :], o_[..., 0, :], rtol=1e-5, atol=1e-6), "mean differs"

    # 3. scores from the oracle's pooled features rounded to fp32 (both sides)
    pq32 = torch.from_numpy(pq_o.astype(np.float32))
    pk32 = torch.from_numpy(pk_o.astype(np.float32))
    wq, wk = inp.wq[hs].contiguous(), inp.wk[hs].contiguous()
    S_g = V.block_scores(pq32.to(DEV), pk32.to(DEV), wq.to(DEV), wk.to(DEV))
    S_o = O.scores(pq32.double().numpy(), pk32.double().numpy(), P.f64(wq), P.f64(wk))
    err = P.score_errors(P.f64(S_g), S_o)
    assert err <= P.SCORE_RTOL, f"score error {err}"

    # 4. selection on the GPU's fp32 scores: bit-exact against the oracle's selection
    sub = synth.head_subset(w, hs)
    sub_maps = V.build_tile_map(sub.grid, sub.head_shapes, sub.n_tail,
                                None if orders is None else orders[hs]).to(DEV)
    lists_g = V.select_blocks(S_g, sub_maps, w.rho)
    V.check_device_status()
    S_g64 = P.f64(S_g)
    lists_o = O.select(S_g64, nv[hs], seg[hs], [nTh[h] for h in hs], w.rho)
    bad, total = P.gpu_lists_equal(lists_g, lists_o, range(len(hs)), rows)
    assert bad == 0, f"{bad}/{total} block lists differ"
    # budget invariants on the GPU lists
    fc = lists_g.full_cnt.cpu().numpy() + lists_g.part_cnt.cpu().numpy()
    for j, h in enumerate(hs):
        k = O.budgets(nTh[h], seg[h], w.rho).sum(axis=1)
        assert (fc[:, j, :nTh[h]] == k[None, :]).all()

    # 5. attention with the oracle's lists (selection on the oracle's fp64 scores)
    lists_ref = O.select(S_o, nv[hs], seg[hs], [nTh[h] for h in hs], w.rho)
    stride = V.list_stride_for(w.nT, w.rho)
    lists_dev = P.lists_to_device(lists_ref, w.B, len(hs), w.nT, stride, DEV)
    qs = torch.from_numpy(oq).to(torch.bfloat16).to(DEV)
    ks = torch.from_numpy(ok_).to(torch.bfloat16).to(DEV)
    vs = torch.from_numpy(ov_).to(torch.bfloat16).to(DEV)
    o_g, lse_g = V.block_sparse_attn_fwd(qs, ks, vs, sub_maps, lists_dev, P.SCALE)
    V.check_device_status()
    todo = attn_rows or [(b, j, r) for b in range(w.B) for j in range(len(hs)) for r in range(w.nT)]
    o_o, lse_o = O.attention(oq, ok_, ov_, nv[hs], lists_ref, P.SCALE, rows=todo)
    o_g64, lse_g64 = P.f64(o_g), P.f64(lse_g)
    diffs, lse_d = [], []
    for (b, j, r) in todo:
        sl = slice(r * 128, (r + 1) * 128)
        if r >= nTh[hs[j]]:
            assert (o_g64[b, j, sl] == 0).all() and np.isneginf(lse_g64[b, j, sl]).all()
            continue
        diffs.append(np.abs(o_g64[b, j, sl] - o_o[b, j, sl]))
        lse_d.append(np.abs(lse_g64[b, j, sl] - lse_o[b, j, sl]).max())
    d = np.concatenate([x.ravel() for x in diffs])
    assert d.max() <= P.ATTN_MAX_ABS and d.mean() <= P.ATTN_MEAN_ABS, (d.max(), d.mean())
    assert max(lse_d) < 2e-3

    # 6. unpermute of a seeded random tile tensor: bit-exact on valid rows
    g = torch.Generator().manual_seed(99)
    ot = torch.randn((w.B, w.H, w.Npad, 128), generator=g).to(torch.bfloat16)
    o_r = V.unpermute(ot.to(DEV), maps, w.N)
    V.check_device_status()
    ref = O.unpermute(P.f64(ot[:, hs]), slots[hs], w.N)
    assert np.array_equal(P.f64(o_r[:, :, hs]), ref), "unpermute differs"
    return dict(d_max=float(d.max()), d_mean=float(d.mean()), score_err=err)


def test_stages_tiny():
    _stage_run(synth.TINY)


def test_stages_small():
    _stage_run(synth.SMALL)


def test_stages_mixed_segments_and_shuffled_heads():
    rng = np.random.default_rng(4)
    heads = [0, 5, 16, 27]
    rows = [(0, j, int(r)) for j in range(4) for r in rng.choice(229, 12, replace=False)]
    rows += [(0, j, r) for j in range(4) for r in (224, 228)]     # audio query tiles
    _stage_run(synth.MIXED, heads=heads, attn_rows=rows)


def test_stages_ragged_heads_and_empty_rows():
    # three tile shapes give 5, 6 and 8 tiles per head: rows past a head's tiles are empty,
    # the grid is padded in t, and the tail makes a partial last tile
    w = synth.Workload("ragged", 9, B=2, H=3, grid=(5, 8, 16),
                       head_shapes=((1, 8, 16), (2, 8, 8), (4, 4, 8)), n_tail=77,
                       rho=((1, 3), (1, 2)))
    _stage_run(w)


@pytest.mark.parametrize("r", [1, 8, 63, 64, 65, 127])
def test_partial_key_tiles_at_the_half_width_boundary(r):
    """Key tiles with at most 64 valid slots take the half-width path (Q K^T and P V over
    their first 64 keys, the softmax over 8 column groups), tiles with more the whole tile.
    Grid 2 x 1 x (128 + r) in (1, 1, 128) tiles gives key tiles of 128, r, 128, r valid slots;
    at density 1 every query tile (whole or partial) visits all four, so both paths alternate
    inside every item."""
    w = synth.Workload(f"halfw{r}", 13, B=1, H=2, grid=(2, 1, 128 + r),
                       head_shapes=((1, 1, 128), (1, 1, 128)), rho=((1, 1),), field=False)
    _stage_run(w)


def test_stages_length_sweep_shortest():
    _stage_run(synth.sweep_length(5), heads=[0, 17, 39],
               attn_rows=[(0, j, r) for j in range(3) for r in (0, 1, 40, 79)])


@pytest.mark.parametrize("B,H,nT", [(1, 1, 1), (2, 3, 5), (1, 2, 129), (1, 4, 300)])
def test_block_scores_tensor_core_split_precision(B, H, nT):
    """The score step runs on the tensor cores as three tf32 products of split operands
    (hi + lo). One tf32 product alone misses the 1e-3 bound (~2e-3 on these inputs); the
    split keeps the error near fp32 rounding, checked here at 2e-5 against the oracle on
    ragged tile counts (one tile, a partial 128-row tile, several tiles)."""
    V = P.veda()
    g = torch.Generator().manual_seed(4242 + nT)
    pq = torch.randn((B, H, nT, 3, 128), generator=g)
    pk = torch.randn((B, H, nT, 3, 128), generator=g)
    wq = 0.02 * torch.randn((H, 128, 384), generator=g)
    wk = 0.02 * torch.randn((H, 128, 384), generator=g)
    S_g = V.block_scores(pq.to(DEV), pk.to(DEV), wq.to(DEV), wk.to(DEV))
    V.check_device_status()
    S_o = O.scores(P.f64(pq), P.f64(pk), P.f64(wq), P.f64(wk))
    err = P.score_errors(P.f64(S_g), S_o)
    assert err <= 2e-5, err


def test_full_density_equals_dense_attention():
    # at 100% density the tiled sparse path (whole public API) is dense softmax attention
    V = P.veda()
    w = synth.Workload("dense", 10, B=1, H=2, grid=(3, 9, 20),
                       head_shapes=((1, 8, 16), (2, 8, 8)), rho=((1, 1),), field=False)
    inp = synth.make_inputs(w)
    maps = V.build_tile_map(w.grid, w.head_shapes).to(DEV)
    bufs = V.sparse_attention(inp.q.to(DEV), inp.k.to(DEV), inp.v.to(DEV), inp.wq.to(DEV),
                              inp.wk.to(DEV), maps, w.rho, P.SCALE)
    V.check_device_status()
    od, _ = O.dense_attention_raster(P.f64(inp.q), P.f64(inp.k), P.f64(inp.v), P.SCALE)
    dmax, dmean = P.attn_errors(P.f64(bufs.o), od)
    assert dmax <= P.ATTN_MAX_ABS and dmean <= P.ATTN_MEAN_ABS, (dmax, dmean)


def test_attention_rescales_when_the_row_maximum_grows():
    """Scores built so that every listed key tile raises a row's maximum by ~64 (log2 units)
    over the previous one (and, for the other half of the rows, lowers it): the kernel must
    move its reference and rescale O each time (without rescaling, P would reach 2^190 and
    overflow fp32). Key tiles 0-2 are full, tile 3 holds 64 valid slots (partial list)."""
    V = P.veda()
    grid, shape = (1, 8, 56), (1, 8, 16)
    maps = V.build_tile_map(grid, [shape]).to(DEV)
    slots, nv, seg, nTh = P.oracle_maps(synth.Workload("growth", 11, B=1, H=1, grid=grid, head_shapes=(shape,),
                                                       rho=((1, 1),), field=False), None)
    nT = int(nTh[0])
    assert nT == 4 and list(nv[0]) == [128, 128, 128, 64]
    g = torch.Generator().manual_seed(11011)
    Npad = nT * 128
    sign = torch.ones(128)
    sign[64:] = -1.0
    q = sign[:, None] + 0.05 * torch.randn((nT, 128, 128), generator=g)          # [tile, row, d]
    c = torch.tensor([0.0, 500.0, 1000.0, 1500.0])                                # score level of key tile j
    k = (c[:, None, None] / 128.0) + 0.5 * torch.randn((nT, 128, 128), generator=g)
    v = torch.randn((nT, 128, 128), generator=g)
    q, k, v = (x.reshape(1, 1, Npad, 128).to(torch.bfloat16) for x in (q, k, v))
    valid = torch.from_numpy(slots[0] >= 0)
    k[0, 0, ~valid] = 0
    v[0, 0, ~valid] = 0
    q[0, 0, ~valid] = 0
    # the construction does what it claims: consecutive listed tiles grow by > 30 (log2)
    qf, kf = P.f64(q)[0, 0], P.f64(k)[0, 0]
    s2 = (qf[:64] @ kf.T) * P.SCALE * math.log2(math.e)
    row_max = [s2[:, j * 128:j * 128 + int(nv[0][j])].max(axis=1) for j in range(nT)]
    assert all((row_max[j + 1] - row_max[j]).min() > 30 for j in range(nT - 1))
    assert (row_max[-1] - row_max[0]).min() > 128
    full = [[[np.arange(3, dtype=np.int64) for _ in range(nT)]]]
    part = [[[np.array([3], dtype=np.int64) for _ in range(nT)]]]
    lists = O.BlockLists(full, part)
    stride = V.list_stride_for(nT, [(1, 1)])
    o_g, lse_g = V.block_sparse_attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), maps, P.lists_to_device(lists, 1, 1, nT, stride, DEV),
                                         P.SCALE)
    V.check_device_status()
    o_o, lse_o = O.attention(P.f64(q), P.f64(k), P.f64(v), nv, lists, P.SCALE)
    og, lg = P.f64(o_g), P.f64(lse_g)
    assert np.isfinite(og).all() and np.isfinite(lg).all()
    d = np.abs(og - o_o)
    assert d.max() <= P.ATTN_MAX_ABS and d.mean() <= P.ATTN_MEAN_ABS, (d.max(), d.mean())
    assert np.all(np.abs(lg - lse_o) <= 2e-3 + 1e-5 * np.abs(lse_o)), np.abs(lg - lse_o).max()


def _end_to_end(w, heads=None, rows=None, attn_rows=None):
    """Public API on the whole workload; every intermediate checked on some heads."""
    V = P.veda()
    inp = synth.make_inputs(w)
    orders = inp.tile_order
    slots, nv, seg, nTh = P.oracle_maps(w, orders)
    maps = V.build_tile_map(w.grid, w.head_shapes, w.n_tail, orders).to(DEV)
    bufs = V.sparse_attention(inp.q.to(DEV), inp.k.to(DEV), inp.v.to(DEV), inp.wq.to(DEV),
                              inp.wk.to(DEV), maps, w.rho, P.SCALE)
    V.check_device_status()
    hs = list(range(w.H)) if heads is None else list(heads)
    q64, k64, v64 = (P.f64(t[:, :, hs]) for t in (inp.q, inp.k, inp.v))
    qt, kt, vt = (O.permute(x, slots[hs]) for x in (q64, k64, v64))
    assert np.array_equal(P.f64(bufs.q_t[:, hs]), qt)
    pq, pk = O.pool(qt, nv[hs]), O.pool(kt, nv[hs])
    assert np.allclose(P.f64(bufs.pooled_q[:, hs]), pq, rtol=1e-5, atol=1e-6)
    assert np.allclose(P.f64(bufs.pooled_k[:, hs]), pk, rtol=1e-5, atol=1e-6)
    S_o = O.scores(pq, pk, P.f64(inp.wq[hs]), P.f64(inp.wk[hs]))
    S_g = P.f64(bufs.scores[:, hs])
    err = P.score_errors(S_g, S_o)
    assert err <= P.SCORE_RTOL, err
    lists_o = O.select(S_g, nv[hs], seg[hs], [nTh[h] for h in hs], w.rho)
    bad, total = P.gpu_lists_equal(bufs.lists, lists_o, hs, rows)
    assert bad == 0, f"{bad}/{total} lists differ"
    # how often does fp64 selection pick differently (near-ties)? reported, not asserted
    lists_64 = O.select(S_o, nv[hs], seg[hs], [nTh[h] for h in hs], w.rho)
    bad64, _ = P.gpu_lists_equal(bufs.lists, lists_64, hs, rows)
    todo = attn_rows or [(b, j, r) for b in range(w.B) for j in range(len(hs)) for r in range(nTh[hs[j]])]
    o_t, _ = O.attention(qt, kt, vt, nv[hs], lists_o, P.SCALE, rows=todo)
    o_g = P.f64(bufs.o_t[:, hs])
    diffs = [np.abs(o_g[b, j, r * 128:(r + 1) * 128] - o_t[b, j, r * 128:(r + 1) * 128]) for (b, j, r) in todo]
    d = np.concatenate([x.ravel() for x in diffs])
    assert d.max() <= P.ATTN_MAX_ABS and d.mean() <= P.ATTN_MEAN_ABS, (d.max(), d.mean())
    # raster output = unpermute of the tiled output (valid slots of the checked heads)
    o_r = P.f64(bufs.o[:, :, hs])
    assert np.array_equal(o_r, O.unpermute(P.f64(bufs.o_t[:, hs]), slots[hs], w.N))
    return dict(lists_fp64_mismatch=bad64, total=total)


def test_host_pipeline_matches_separate_calls():
    """Three different clips through the HostPipeline (two slots, so one is reused while its
    neighbour is in flight) give the outputs of separate sparse_attention calls bit for bit."""
    V = P.veda()
    w = synth.SMALL
    inp = synth.make_inputs(w)
    maps = V.build_tile_map(w.grid, w.head_shapes, w.n_tail, inp.tile_order).to(DEV)
    g = torch.Generator().manual_seed(77)
    clips = []
    for i in range(3):
        q = (inp.q.float() * (1.0 + 0.5 * i)).to(torch.bfloat16)
        k = (inp.k.float() + 0.1 * i).to(torch.bfloat16)
        v = torch.randn(inp.v.shape, generator=g).to(torch.bfloat16)
        clips.append((q, k, v))
    B, N, H, D = inp.q.shape
    pipe = V.HostPipeline(B, N, H, maps, w.rho, P.SCALE, torch.device(DEV), depth=2)
    outs = [torch.empty((B, N, H, D), dtype=torch.bfloat16).pin_memory() for _ in clips]
    wq, wk = inp.wq.pin_memory(), inp.wk.pin_memory()
    for (q, k, v), o in zip(clips, outs):
        pipe.submit(q.pin_memory(), k.pin_memory(), v.pin_memory(), wq, wk, o)
    pipe.synchronize()
    V.check_device_status()
    for (q, k, v), o in zip(clips, outs):
        ref = V.sparse_attention(q.to(DEV), k.to(DEV), v.to(DEV), inp.wq.to(DEV), inp.wk.to(DEV), maps,
                                 w.rho, P.SCALE)
        assert torch.equal(o, ref.o.cpu())


def test_end_to_end_tiny():
    _end_to_end(synth.TINY)


def test_end_to_end_small():
    r = _end_to_end(synth.SMALL)
    assert r["lists_fp64_mismatch"] <= r["total"] // 20


def test_end_to_end_clip16x9_full_size():
    # the benchmark's workload and launch configuration; sampled heads and query tiles
    rng = np.random.default_rng(3)
    heads = [0, 13, 39]
    rows = [int(r) for r in rng.choice(496, 40, replace=False)] + [0, 1, 495]
    attn = [(0, j, r) for j in range(3) for r in rows[:8] + [0, 495]]
    r = _end_to_end(synth.CLIP16x9, heads=heads, rows=rows, attn_rows=attn)
    assert r["lists_fp64_mismatch"] <= r["total"] // 10


def test_device_check_flags_bad_lists_without_fault():
    # an out-of-range key index is caught by the kernel's own bounds check: it reads a
    # valid tile instead, records VEDA_ERR_DEVICE_CHECK and the call returns normally
    V = P.veda()
    w = synth.TINY
    inp = synth.make_inputs(w)
    maps = V.build_tile_map(w.grid, w.head_shapes).to(DEV)
    bufs = V.sparse_attention(inp.q.to(DEV), inp.k.to(DEV), inp.v.to(DEV), inp.wq.to(DEV),
                              inp.wk.to(DEV), maps, w.rho, P.SCALE)
    V.check_device_status()
    bufs.lists.full_idx[0, 0, 1, 0] = 1000
    V.block_sparse_attn_fwd(bufs.q_t, bufs.k_t, bufs.v_t, maps, bufs.lists, P.SCALE)
    with pytest.raises(V.VedaError) as e:
        V.check_device_status()
    assert e.value.status == 5
    V.check_device_status()       # the word was cleared


@pytest.mark.parametrize("name,heads,rows", [
    ("clip16x9_rho1_1", [7], [0, 250, 495]),          # 100% density: dense attention
    ("clip16x9_rho1_2", [3], [1, 300]),
    ("clip16x9_rho1_5", [30], [2, 251, 494]),         # 20%: rows of 99 and 100 key tiles
    ("clip16x9_rho1_20", [21], [0, 123, 495]),        # 5%: rows of 24 and 25 key tiles
    ("len_T15", [5, 38], [0, 120, 239]),              # 24k tokens, nT = 240
    ("len_T62", [11], [0, 500, 991]),                 # 100k tokens, nT = 992
])
def test_sweep_extremes_sampled(name, heads, rows):
    w = synth.get(name)
    attn = [(0, 0, r) for r in rows]
    _end_to_end(w, heads=heads, rows=rows, attn_rows=attn)


def test_stages_length_sweep_24k():
    # the 24k-token point of the length sweep (15 frames of 30 x 54, nT = 240), stage by stage
    _stage_run(synth.sweep_length(15), heads=[0, 22, 39],
               attn_rows=[(0, j, r) for j in range(3) for r in (0, 1, 119, 239)])


def test_density_one_twentieth_rows_of_only_the_diagonal():
    """Density 1/20 over 32 key tiles is 1.6 tiles per row: Bresenham gives rows of 1 and 2
    tiles, and a row whose budget is 1 holds its own (diagonal) tile alone. Checked stage by
    stage and end to end against the oracle, then row by row on the GPU's lists."""
    V = P.veda()
    w = synth.Workload("short_rho1_20", 12, B=1, H=4, grid=(2, 30, 54),
                       head_shapes=((1, 8, 16),) * 4, rho=((1, 20),))
    assert w.nT == 32
    _stage_run(w)
    _end_to_end(w)
    inp = synth.make_inputs(w)
    slots, nv, seg, nTh = P.oracle_maps(w, None)
    maps = V.build_tile_map(w.grid, w.head_shapes).to(DEV)
    bufs = V.sparse_attention(inp.q.to(DEV), inp.k.to(DEV), inp.v.to(DEV), inp.wq.to(DEV),
                              inp.wk.to(DEV), maps, w.rho, P.SCALE)
    V.check_device_status()
    k = O.budgets(nTh[0], seg[0], w.rho).sum(axis=1)
    ones = np.flatnonzero(k == 1)
    assert len(ones) >= 10 and set(k.tolist()) == {1, 2}
    fc, fi = bufs.lists.full_cnt.cpu().numpy(), bufs.lists.full_idx.cpu().numpy()
    pc, pi = bufs.lists.part_cnt.cpu().numpy(), bufs.lists.part_idx.cpu().numpy()
    for h in range(w.H):
        for r in ones:
            got = sorted(fi[0, h, r, :fc[0, h, r]].tolist() + pi[0, h, r, :pc[0, h, r]].tolist())
            assert got == [r], (h, r, got)


def test_maximum_tile_count():
    """The largest tile count the selection accepts (2,048 tiles per head: 128 frames of 30 x 54,
    207,360 tokens), stage by stage on two heads: selection on every row (its per-warp shared
    memory is then above the default 48 KB a launch gets), attention on sampled query tiles."""
    w = synth.Workload("max_tiles", 13, B=1, H=2, grid=(128, 30, 54), head_shapes=((1, 8, 16),) * 2)
    assert w.nT == 2048
    _stage_run(w, attn_rows=[(0, j, r) for j in range(2) for r in (0, 1, 1023, 2046, 2047)])


def test_density_zero_keeps_only_the_diagonal():
    """Density 0: every budget is 0 but the query's own segment, which the forced diagonal
    raises to 1, so every row's list is its own tile and attention stays inside the tile."""
    V = P.veda()
    w = synth.Workload("rho0", 14, B=1, H=3, grid=(6, 17, 40), head_shapes=((1, 8, 16), (2, 8, 8), (4, 4, 8)),
                       rho=((0, 1),))
    _stage_run(w)
    inp = synth.make_inputs(w)
    maps = V.build_tile_map(w.grid, w.head_shapes).to(DEV)
    bufs = V.sparse_attention(inp.q.to(DEV), inp.k.to(DEV), inp.v.to(DEV), inp.wq.to(DEV),
                              inp.wk.to(DEV), maps, w.rho, P.SCALE)
    V.check_device_status()
    slots, nv, seg, nTh = P.oracle_maps(w, None)
    fc, fi = bufs.lists.full_cnt.cpu().numpy(), bufs.lists.full_idx.cpu().numpy()
    pc, pi = bufs.lists.part_cnt.cpu().numpy(), bufs.lists.part_idx.cpu().numpy()
    for h in range(w.H):
        for r in range(w.nT):
            got = sorted(fi[0, h, r, :fc[0, h, r]].tolist() + pi[0, h, r, :pc[0, h, r]].tolist())
            assert got == ([r] if r < nTh[h] else []), (h, r, got)


def test_bounded_wait_runs_out_and_context_survives():
    # failure detection without a fault: a wait on a barrier nothing arrives on gives up
    # after 2 ms, the status word says VEDA_ERR_TIMEOUT, and the next call works
    V = P.veda()
    V.check_device_status()
    V.selftest_wait_timeout(2000)
    with pytest.raises(V.VedaError) as e:
        V.check_device_status()
    assert e.value.status == 4
    V.check_device_status()
    _stage_run(synth.TINY)


@pytest.mark.parametrize("w", [synth.TINY, synth.SMALL, synth.MIXED], ids=lambda w: w.name)
def test_fused_permute_pool(w):
    """Steps 1 + 2 fused: tiles bit-identical to the permute, max / min identical to the
    oracle's pooling, mean within 1e-5 relative (fp32 summation order)."""
    V = P.veda()
    inp = synth.make_inputs(w)
    orders = inp.tile_order
    slots, nv, seg, nTh = P.oracle_maps(w, orders)
    maps = V.build_tile_map(w.grid, w.head_shapes, w.n_tail, orders).to(DEV)
    for x in (inp.q, inp.k):
        xd = x.to(DEV)
        xt, pooled = V.permute_pool(xd, maps)
        V.check_device_status()
        assert torch.equal(xt, V.permute_tiles(xd, maps)), "fused tiles differ from the permute"
        ref = O.pool(O.permute(P.f64(x), slots), nv)
        g = P.f64(pooled)
        assert np.array_equal(g[..., 1:, :], ref[..., 1:, :]), "max/min differ"
        assert np.allclose(g[..., 0, :], ref[..., 0, :], rtol=1e-5, atol=1e-6), "mean differs"
