"""GPU parity of the block-sparse attention backward and the transposed lists, through the C ABI.

The GPU runs its own chain (permute, pool, scores, selection, forward for O and LSE,
transposed lists, backward) on seeded inputs and a seeded output gradient dO; the oracle
runs its own fp64 chain from the same bf16 bytes with the GPU's block lists (fed back as
the parity rule feeds the selection its scores). Transposed lists are compared bit-exactly.
Gradient tolerance (derived): P and dS enter the tensor cores as bf16 (relative 2^-9 per
element), D uses the bf16 forward output, and the sums run in fp32 over thousands of keys,
so per tensor max |gpu - ref| <= 2e-2 max |ref| and mean |gpu - ref| <= 2e-3 max |ref|
(the forward's bounds, relative to the gradient's scale), over valid slots only.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import veda_oracle as O
import parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
MAX_REL, MEAN_REL = 2e-2, 2e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from block_sparse_attention_max_b200 import build
    build.build()
    V = P.veda()
    V.lib()
    yield
    V.check_device_status()


def _oracle_lists(gl, heads):
    fc, fi = gl.full_cnt.cpu().numpy(), gl.full_idx.cpu().numpy()
    pc, pi = gl.part_cnt.cpu().numpy(), gl.part_idx.cpu().numpy()
    B, _, nT = fc.shape
    full = [[[fi[b, h, r, :fc[b, h, r]].astype(np.int64) for r in range(nT)] for h in heads] for b in range(B)]
    part = [[[pi[b, h, r, :pc[b, h, r]].astype(np.int64) for r in range(nT)] for h in heads] for b in range(B)]
    return O.BlockLists(full, part)


def _run(w, heads):
    V = P.veda()
    inp = synth.make_inputs(w)
    orders = inp.tile_order
    slots, nv, seg, nTh = P.oracle_maps(w, orders)
    maps = V.build_tile_map(w.grid, w.head_shapes, w.n_tail, orders).to(DEV)
    q_d, k_d, v_d, wq, wk = (t.to(DEV) for t in (inp.q, inp.k, inp.v, inp.wq, inp.wk))
    bufs = V.sparse_attention(q_d, k_d, v_d, wq, wk, maps, w.rho, P.SCALE)
    gen = torch.Generator().manual_seed(1000 * w.wid + 8)
    dout = torch.randn(inp.q.shape, generator=gen).to(torch.bfloat16)
    do_t = V.permute_tiles(dout.to(DEV), maps)
    tl = V.transpose_lists(bufs.lists, maps)
    dq, dk, dv = V.block_sparse_attn_bwd(bufs.q_t, bufs.k_t, bufs.v_t, bufs.o_t, do_t, bufs.lse, maps,
                                         bufs.lists, tl, P.SCALE)
    V.check_device_status()

    B, H, Npad, D = bufs.q_t.shape
    nT = Npad // 128
    lists_o = _oracle_lists(bufs.lists, list(range(H)))
    # transposed lists: bit-exact
    T = O.transpose_lists(lists_o, nTh, nT)
    tc, ti = tl.cnt.cpu().numpy(), tl.idx.cpu().numpy()
    for b in range(B):
        for h in range(H):
            for j in range(nT):
                assert tc[b, h, j] == len(T[b][h][j]) and np.array_equal(ti[b, h, j, :tc[b, h, j]], T[b][h][j])

    # gradients of the checked heads against the oracle's own forward and backward
    lists_h = _oracle_lists(bufs.lists, heads)
    qt = O.permute(P.f64(inp.q[:, :, heads]), slots[heads])
    kt = O.permute(P.f64(inp.k[:, :, heads]), slots[heads])
    vt = O.permute(P.f64(inp.v[:, :, heads]), slots[heads])
    dot = O.permute(P.f64(dout[:, :, heads]), slots[heads])
    o_o, lse_o = O.attention(qt, kt, vt, nv[heads], lists_h, P.SCALE)
    gq, gk, gv = O.attention_backward(qt, kt, vt, nv[heads], lists_h, P.SCALE, np.nan_to_num(o_o),
                                      np.nan_to_num(lse_o, neginf=0.0), dot)
    for name, g_gpu, g_ref in (("dq", dq, gq), ("dk", dk, gk), ("dv", dv, gv)):
        g = P.f64(g_gpu[:, heads])
        for j in range(len(heads)):
            ok = slots[heads[j]] >= 0                      # valid slots of the head
            d = np.abs(g[:, j][:, ok] - g_ref[:, j][:, ok])
            scale = np.abs(g_ref[:, j][:, ok]).max()
            assert d.max() <= MAX_REL * scale, f"{name} head {heads[j]}: max err {d.max():.3g} vs {scale:.3g}"
            assert d.mean() <= MEAN_REL * scale, f"{name} head {heads[j]}: mean err {d.mean():.3g} vs {scale:.3g}"
            # pad key slots get no gradient
            if name in ("dk", "dv"):
                assert not g[:, j][:, ~ok].any()


def test_backward_tiny():
    _run(synth.TINY, [0, 1])


def test_backward_small():
    _run(synth.SMALL, [0, 6])


def test_backward_mixed_shapes_tail_and_segments():
    _run(synth.MIXED, [17])
