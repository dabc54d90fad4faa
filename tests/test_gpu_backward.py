"""GPU parity of the block-sparse attention backward and the transposed lists, through the C ABI.

The GPU runs its own chain (permute, pool, scores, selection, forward for O and LSE,
transposed lists, backward) on seeded inputs and a seeded output gradient dO; the oracle
runs its own fp64 chain from the same bf16 bytes with the GPU's block lists (fed back as
the parity rule feeds the selection its scores). Transposed lists are compared bit-exactly.

Two gradient checks per case:
- Backward alone: as in the stage tests, the GPU backward is fed the oracle's own forward
  output (O rounded to the bf16 tensor it is, reading R16, and the fp32 LSE) on the checked
  heads. P and dS enter the tensor cores as bf16 (relative 2^-9 per element) and the sums run
  in fp32 over thousands of keys, so per tensor max |gpu - ref| <= 2e-2 max |ref| and
  mean |gpu - ref| <= 2e-3 max |ref| (the forward's bounds, relative to the gradient's
  scale), over valid slots only.
- Forward then backward (the GPU's own O and LSE): D = rowsum(dO * O) now carries the
  forward's output error eO, eD_i = dO_i . eO_i, and D enters dS = P (dP - D) linearly, so
  dq_i moves by exactly -scale eD_i (P K)_i and dk_j by -scale sum_i P_ij eD_i Q_i, while dv
  does not depend on D. The forward's output is within one bf16 ulp of the exact value plus
  the rounding of P to bf16 before the PV product, |eO_id| <= ulp(O_id) + 2^-8 (P |V|)_id,
  so |eD_i| <= sum_d |dO_id| that bound; the tolerance of dq and dk is the first check's
  plus the band this gives, computed by the oracle (_band). With smooth inputs |D| reaches
  ~30 and the keys a row attends to point the same way, so the band is what dominates dq.
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
    # the backward receives the forward's output, which is a bf16 tensor (reading R16): the
    # oracle's own O, rounded to bf16, enters D = rowsum(dO * O) on both sides
    o_b = torch.from_numpy(np.nan_to_num(o_o)).to(torch.bfloat16).double().numpy()
    lse_b = np.where(np.isfinite(lse_o), lse_o, -np.inf)
    ref = O.attention_backward(qt, kt, vt, nv[heads], lists_h, P.SCALE, o_b,
                               np.nan_to_num(lse_o, neginf=0.0), dot)

    # backward alone: the oracle's O and LSE on the checked heads
    o_in, lse_in = bufs.o_t.clone(), bufs.lse.clone()
    o_in[:, heads] = torch.from_numpy(o_b).to(torch.bfloat16).to(DEV)
    lse_in[:, heads] = torch.from_numpy(lse_b).to(torch.float32).to(DEV)
    alone = V.block_sparse_attn_bwd(bufs.q_t, bufs.k_t, bufs.v_t, o_in, do_t, lse_in, maps,
                                    bufs.lists, tl, P.SCALE)
    V.check_device_status()
    zero = [np.zeros_like(r) for r in ref]
    _compare(alone, ref, zero, heads, slots, "alone")

    # forward then backward: the band of the forward's output error through D
    _compare((dq, dk, dv), ref, _band(qt, kt, vt, dot, o_b, lse_o, nv[heads], lists_h),
             heads, slots, "chained")


def _band(qt, kt, vt, dot, o_b, lse_o, nv, lists):
    """Largest change of dq and dk from the forward's output error, by the oracle.

    eO_id = ulp(O_id) + 2^-8 (P |V|)_id bounds the output error and eD_i = sum_d |dO_id| eO_id
    the error of D_i; dq_i moves by scale eD_i |(P K)_i| and dk_j by at most
    scale sum_i P_ij eD_i |Q_i|, which is the dV of a backward whose output gradient is
    eD_i |Q_i| (dV = P^T dO)."""
    m, e = np.frexp(np.abs(o_b))
    ulp = np.where(o_b != 0, np.ldexp(1.0, e - 8), 0.0)       # bf16 ulp of |O|, |O| = m 2^e
    pav, _ = O.attention(qt, kt, np.abs(vt), nv, lists, P.SCALE)
    e_o = ulp + 2.0 ** -8 * np.nan_to_num(pav)
    e_d = (np.abs(dot) * e_o).sum(axis=-1)                     # [B, H, Npad]
    pk, _ = O.attention(qt, kt, kt, nv, lists, P.SCALE)
    band_q = P.SCALE * e_d[..., None] * np.abs(np.nan_to_num(pk))
    _, _, pq = O.attention_backward(qt, kt, vt, nv, lists, P.SCALE, np.zeros_like(o_b),
                                    np.nan_to_num(lse_o, neginf=0.0), e_d[..., None] * np.abs(qt))
    band_k = P.SCALE * pq
    return band_q, band_k, np.zeros_like(band_q)


def _compare(got, ref, band, heads, slots, what):
    for name, g_gpu, g_ref, b_ in zip(("dq", "dk", "dv"), got, ref, band):
        g = P.f64(g_gpu[:, heads])
        for j in range(len(heads)):
            ok = slots[heads[j]] >= 0                      # valid slots of the head
            d = np.abs(g[:, j][:, ok] - g_ref[:, j][:, ok])
            extra = b_[:, j][:, ok]
            top = np.abs(g_ref[:, j][:, ok]).max()
            assert np.all(d <= MAX_REL * top + extra), \
                f"{what} {name} head {heads[j]}: max err {d.max():.3g} vs {top:.3g} (band {extra.max():.3g})"
            assert d.mean() <= MEAN_REL * top + extra.mean(), \
                f"{what} {name} head {heads[j]}: mean err {d.mean():.3g} vs {top:.3g}"
            # pad key slots get no gradient
            if name in ("dk", "dv"):
                assert not g[:, j][:, ~ok].any()


def test_backward_tiny():
    _run(synth.TINY, [0, 1])


def test_backward_small():
    _run(synth.SMALL, [0, 6])


def test_backward_mixed_shapes_tail_and_segments():
    _run(synth.MIXED, [17])


def test_backward_ragged_heads_batch_and_empty_rows():
    """Heads with different tile counts (empty lists for rows and key tiles past a head's
    count), two batch entries, partial tiles along w."""
    w = synth.Workload("ragged", 9, B=2, H=3, grid=(5, 8, 16),
                       head_shapes=((1, 8, 16), (2, 8, 8), (4, 4, 8)), n_tail=0,
                       rho=((1, 2),), field="smooth")
    _run(w, [0, 1, 2])


@pytest.mark.parametrize("r", [1, 63, 64, 65])
def test_backward_partial_key_tiles_at_the_half_width_boundary(r):
    """In the dQ pass, key tiles with at most 64 valid slots run S, dP and dQ's accumulation
    over their first 64 keys: tiles of 128, r, 128, r valid slots, density 1, so every item
    mixes both kinds (and the dK/dV pass sees partial query and key tiles of r rows)."""
    w = synth.Workload(f"halfw{r}", 13, B=1, H=2, grid=(2, 1, 128 + r),
                       head_shapes=((1, 1, 128), (1, 1, 128)), rho=((1, 1),), field=False)
    _run(w, [0, 1])


def test_backward_clip16x9_one_head():
    """The 16:9 clip at full size (40 heads launched, the benchmark's configuration), every
    transposed list checked, the gradients of head 0 against the oracle over all its rows."""
    _run(synth.CLIP16x9, [0])


def test_backward_from_two_host_threads_matches_serial():
    """The backward runs dQ on a second stream of the library, forked from and joined back
    into the caller's stream with events the device's calls share. Two host threads, each on
    a stream of its own with its own output gradient, enqueue backward calls at the same
    time; every result equals the serial call's bit for bit (every output tile is reduced
    inside one CTA, so the kernels are deterministic whichever CTA takes an item)."""
    import threading
    V = P.veda()
    w = synth.SMALL
    inp = synth.make_inputs(w)
    maps = V.build_tile_map(w.grid, w.head_shapes, w.n_tail, inp.tile_order).to(DEV)
    bufs = V.sparse_attention(inp.q.to(DEV), inp.k.to(DEV), inp.v.to(DEV), inp.wq.to(DEV), inp.wk.to(DEV),
                              maps, w.rho, P.SCALE)
    tl = V.transpose_lists(bufs.lists, maps)
    grads = []
    for seed in (1, 2):
        g = torch.Generator().manual_seed(5000 + seed)
        grads.append(V.permute_tiles(torch.randn(inp.q.shape, generator=g).to(torch.bfloat16).to(DEV), maps))

    def bwd(do_t):
        return V.block_sparse_attn_bwd(bufs.q_t, bufs.k_t, bufs.v_t, bufs.o_t, do_t, bufs.lse, maps,
                                       bufs.lists, tl, P.SCALE)

    ref = [bwd(grads[i]) for i in range(2)]
    torch.cuda.synchronize()
    V.check_device_status()
    reps = 4
    out = [[None] * reps for _ in range(2)]
    errors = []

    def worker(i):
        try:
            s = torch.cuda.Stream(device=DEV)
            with torch.cuda.device(DEV), torch.cuda.stream(s):
                for r in range(reps):
                    out[i][r] = bwd(grads[i])
            s.synchronize()
        except Exception as e:  # pragma: no cover - reported below
            errors.append(e)

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
    torch.cuda.synchronize()
    V.check_device_status()
    for i in range(2):
        for r in range(reps):
            for got, want in zip(out[i][r], ref[i]):
                assert torch.equal(got, want), (i, r)
