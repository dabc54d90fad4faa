"""Benchmark of the Veda block-sparse attention hot path on B200.

One step = one pass of the whole path (permute Q/K/V, pool Q/K, block scores, block
selection, block-sparse attention, unpermute) over the 16:9-clip workload: B=1, 40
heads, grid 31x30x54 (50,220 tokens), tile (1,8,16), 10% density (90% sparsity).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {veda,reference}]

Prints one JSON line (rank 0). ``value`` is the effective attention throughput of the
whole step: FLOPs of the visited 128x128 blocks (4*128^3 each: Q K^T and P V) divided
by the step time, summed over ranks. Per-kernel times come from CUDA events on the
launching stream inside the timed region. ``--impl reference`` times the fp64 CPU
oracle on a bounded sample of the same workload (the CPU baseline).
Under torchrun (N > 1) every rank runs an independent replica ("replicas only": the
path has no exchange step); time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time
from typing import Optional

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "block-sparse attn ms/call & effective TFLOPS at 90% sparsity; % bf16 peak"
UNIT = "TFLOP/s"
FLOP_PER_BLOCK = 4 * 128 ** 3
WORKLOAD = synth.CLIP16x9
SCALE = 1.0 / math.sqrt(128)


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sus=d["bf16_tflops_sustained"],
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, source="fallback")


def _dist(backend: str = "nccl"):
    """One process per GPU, from the torchrun environment (RANK, LOCAL_RANK, WORLD_SIZE,
    MASTER_ADDR/PORT). NCCL on GPUs; the CPU tests of this path use gloo. Short timeout, so
    that ranks waiting for a lost peer end with an error."""
    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        import torch.distributed as dist
        from datetime import timedelta
        local = int(os.environ.get("LOCAL_RANK", "0"))
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=timedelta(seconds=60))
        return dist, dist.get_rank(), dist.get_world_size()
    return None, 0, 1


def _max_over_ranks(dist, x: float, device) -> float:
    """The slowest rank's time (every rank gets it; identity without a process group)."""
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _job_tflops(world: int, flop_per_rank_step: float, ms_step: float) -> float:
    """Whole-job throughput: the work all replicas did over the slowest rank's step time."""
    return world * flop_per_rank_step / (ms_step * 1e-3) / 1e12


class Clocks:
    """nvidia-smi sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int, path: Optional[str] = None):
        self.idx = device_index
        self.proc = None
        self.path = path or os.path.join(tempfile.gettempdir(), f"veda_clocks_rank{device_index}.csv")

    def start(self):
        """Start sampling every 50 ms and return once the first sample is written (at most
        3 s), so that the samples cover the timed region that follows."""
        try:
            d = os.path.dirname(self.path)
            if d:
                os.makedirs(d, exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=self.f, stderr=subprocess.DEVNULL)
            t0 = time.time()
            while time.time() - t0 < 3.0 and self.proc.poll() is None and os.path.getsize(self.path) == 0:
                time.sleep(0.02)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = max(mx, float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        loaded = [s for s in sm if s > 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def _attn_traffic(heads: int):
    """DRAM bytes per attention launch at the 16:9 clip with `heads` heads, from the committed
    ncu record (profiles/attn_fwd_clip16x9.traffic.json: bytes per launch of the captured case
    and its head count; traffic grows with the heads, whose items are independent), or None
    when the kernel source has changed since the counters were taken."""
    import hashlib
    rec = os.path.join(ROOT, "profiles", "attn_fwd_clip16x9.traffic.json")
    src = os.path.join(ROOT, "block_sparse_attention_max_b200", "csrc", "k_attn.cuh")
    if not (os.path.exists(rec) and os.path.exists(src)):
        return None
    try:
        r = json.load(open(rec))
        digest = hashlib.sha256(open(src, "rb").read()).hexdigest()
        if r.get("kernel_source_sha256") != digest:
            return None
        return int(round(r["dram_bytes_per_launch"] * heads / r["heads"]))
    except (OSError, ValueError, KeyError, TypeError, ZeroDivisionError):
        return None


def _attn_algorithmic_bytes(H: int, nT: int, B: int = 1) -> int:
    """Bytes the attention step must move at least: the tiled Q, K and V read once and O
    written once (bf16, 128 x 128 per tile), plus the fp32 LSE row per query slot."""
    tiles = B * H * nT
    return tiles * (4 * 128 * 128 * 2 + 128 * 4)


# Dense bf16 tensor-core work an SM retires per clock: one M128 N128 K16 tcgen05.mma
# (524,288 FLOP) every 64 cycles.
BF16_FLOP_PER_CLK_SM = 8192


def _visited_blocks(lists) -> int:
    return int(lists.full_cnt.sum().item() + lists.part_cnt.sum().item())


def _valid_token_flop(lists, tile_valid: np.ndarray) -> float:
    """Attention FLOP over valid query x valid key pairs of the visited blocks (4 D per pair)."""
    fc, pc = lists.full_cnt.cpu().numpy(), lists.part_cnt.cpu().numpy()
    fi, pi = lists.full_idx.cpu().numpy(), lists.part_idx.cpu().numpy()
    B, H, nT = fc.shape
    total = 0.0
    for h in range(H):
        v = tile_valid[h].astype(np.float64)
        col = np.arange(fi.shape[-1])
        for b in range(B):
            fk = np.where(col[None, :] < fc[b, h][:, None], v[np.clip(fi[b, h], 0, nT - 1)], 0.0).sum(1)
            pk = np.where(col[None, :] < pc[b, h][:, None], v[np.clip(pi[b, h], 0, nT - 1)], 0.0).sum(1)
            total += float((v * (fk + pk)).sum())
    return 4.0 * 128 * total


def _executed_flop(lists, tile_valid: np.ndarray) -> float:
    """Tensor-core FLOP the forward kernel executes: 4 * 128 * 128 * w per visited block, w = 64
    keys for a partial-list key tile with at most 64 valid slots (its upper half is not
    computed), else 128."""
    pc = lists.part_cnt.cpu().numpy()
    pi = lists.part_idx.cpu().numpy()
    B, H, nT = pc.shape
    half = 0
    for h in range(H):
        small = tile_valid[h] <= 64
        col = np.arange(pi.shape[-1])
        for b in range(B):
            sel = col[None, :] < pc[b, h][:, None]
            half += int((sel & small[np.clip(pi[b, h], 0, nT - 1)]).sum())
    return (_visited_blocks(lists) - half / 2.0) * FLOP_PER_BLOCK


def _random_device_lists(rng, lists, tile_valid: np.ndarray, dev):
    """Fresh uniform random block lists with a forced diagonal and the same per-row budget as
    `lists` (the 'new pattern per call' timing), split into full / partial tiles."""
    from block_sparse_attention_max_b200 import veda as V
    kcnt = (lists.full_cnt + lists.part_cnt).cpu().numpy()
    B, H, nT = kcnt.shape
    keys = rng.random((B, H, nT, nT), dtype=np.float32)
    ar = np.arange(nT)
    keys[:, :, ar, ar] = -1.0                                   # the diagonal ranks first
    rank = np.argsort(np.argsort(keys, axis=-1), axis=-1)
    sel = rank < kcnt[..., None]
    full = sel & (tile_valid[None, :, None, :] == 128)
    part = sel & ~full
    stride = lists.stride
    fi = np.argsort(~full, axis=-1, kind="stable")[..., :stride].astype(np.int32)   # ascending
    pi = np.argsort(~part, axis=-1, kind="stable")[..., :stride].astype(np.int32)
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(dev)
    return V.BlockLists(t(full.sum(-1).astype(np.int32)), t(fi), t(part.sum(-1).astype(np.int32)), t(pi), stride)


def run_veda(args):
    from block_sparse_attention_max_b200 import veda as V
    dist, rank, world = _dist()
    dev = torch.device("cuda", torch.cuda.current_device())
    w = workload(args)
    peaks = _peaks()

    inp = synth.make_inputs(w)
    hmaps = V.build_tile_map(w.grid, w.head_shapes, w.n_tail, inp.tile_order)
    maps = hmaps.to(dev)
    q, k, v = (t.to(dev) for t in (inp.q, inp.k, inp.v))
    wq, wk = inp.wq.to(dev), inp.wk.to(dev)
    B, N, H, D = q.shape
    bufs = V.PathBuffers.allocate(B, N, H, maps, w.rho, dev)
    stream = torch.cuda.current_stream()

    ev = {}

    def event():
        return torch.cuda.Event(enable_timing=True)

    def step(record: bool):
        marks = [event() for _ in range(7)] if record else None
        if record:
            marks[0].record(stream)
        # steps 1 + 2 of Q and K in one pass each (the fused call), step 1 of V
        V.permute_pool(q, maps, bufs.q_t, bufs.pooled_q)
        V.permute_pool(k, maps, bufs.k_t, bufs.pooled_k)
        if record:
            marks[1].record(stream)
        V.permute_tiles(v, maps, bufs.v_t)
        if record:
            marks[2].record(stream)
        V.block_scores(bufs.pooled_q, bufs.pooled_k, wq, wk, bufs.scores, bufs.workspace)
        if record:
            marks[3].record(stream)
        V.select_blocks(bufs.scores, maps, w.rho, bufs.lists.stride, bufs.lists)
        if record:
            marks[4].record(stream)
        V.block_sparse_attn_fwd(bufs.q_t, bufs.k_t, bufs.v_t, maps, bufs.lists, SCALE, bufs.o_t, bufs.lse)
        if record:
            marks[5].record(stream)
        V.unpermute(bufs.o_t, maps, N, bufs.o)
        if record:
            marks[6].record(stream)
        return marks

    for _ in range(args.warmup):
        step(False)
    V.check_device_status()
    blocks = _visited_blocks(bufs.lists)
    flop_step = blocks * FLOP_PER_BLOCK
    launches_per_step = 2 + 1 + 2 + 1 + 1 + 1

    clocks = Clocks(dev.index, args.clocks_csv)
    clocks.start()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    t0, t1 = event(), event()
    t0.record(stream)
    all_marks = [step(True) for _ in range(args.steps)]
    t1.record(stream)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clk = clocks.stop()
    V.check_device_status()
    ms_total = t0.elapsed_time(t1)
    stage_names = ["permute_pool_qk", "permute_v", "scores", "select", "attention", "unpermute"]
    stage_ms = {n: statistics.mean(m[i].elapsed_time(m[i + 1]) for m in all_marks)
                for i, n in enumerate(stage_names)}
    ms_total = _max_over_ranks(dist, ms_total, dev)
    ms_step = ms_total / args.steps

    # end-to-end through the public API with host buffers (pinned): every step copies its
    # inputs to the device and its output back inside the timed region; the HostPipeline
    # overlaps step i's compute with the copies of steps i + 1 (in) and i - 1 (out)
    qh, kh, vh = (t.pin_memory() for t in (inp.q, inp.k, inp.v))
    wqh, wkh = inp.wq.pin_memory(), inp.wk.pin_memory()
    oh = torch.empty((B, N, H, D), dtype=torch.bfloat16).pin_memory()
    pipe = V.HostPipeline(B, N, H, maps, w.rho, SCALE, dev, depth=2)
    for _ in range(max(2, args.warmup // 2)):
        pipe.submit(qh, kh, vh, wqh, wkh, oh)
    pipe.synchronize()
    e_steps = max(3, min(args.steps, 10))
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = event(), event()
    e0.record(pipe.h2d)
    for _ in range(e_steps):
        pipe.submit(qh, kh, vh, wqh, wkh, oh)
    e1.record(pipe.d2h)
    torch.cuda.synchronize()
    e_ms = _max_over_ranks(dist, e0.elapsed_time(e1) / e_steps, dev)
    V.check_device_status()
    h2d = sum(t.numel() * t.element_size() for t in (qh, kh, vh, wqh, wkh))
    d2h = oh.numel() * oh.element_size()

    attn_ms = stage_ms["attention"]
    attn_tflops = flop_step / (attn_ms * 1e-3) / 1e12

    # secondary attention figures: valid-token and dense-equivalent rates of the same calls,
    # and the same kernel on fresh uniform random lists (same budgets), one pattern per call
    tile_valid = np.asarray(hmaps.tile_valid)
    valid_flop = _valid_token_flop(bufs.lists, tile_valid)
    exec_flop = _executed_flop(bufs.lists, tile_valid)
    rng = np.random.default_rng(7007)
    patterns = [_random_device_lists(rng, bufs.lists, tile_valid, dev) for _ in range(4)]
    rnd_blocks = statistics.mean(_visited_blocks(p) for p in patterns)
    for p in patterns:
        V.block_sparse_attn_fwd(bufs.q_t, bufs.k_t, bufs.v_t, maps, p, SCALE, bufs.o_t, bufs.lse)
    rnd_times = []
    for i in range(max(3, min(args.steps, 12))):
        a0, a1 = event(), event()
        a0.record(stream)
        V.block_sparse_attn_fwd(bufs.q_t, bufs.k_t, bufs.v_t, maps, patterns[i % len(patterns)], SCALE,
                                bufs.o_t, bufs.lse)
        a1.record(stream)
        a1.synchronize()
        rnd_times.append(a0.elapsed_time(a1))
    V.check_device_status()
    rnd_ms = statistics.median(rnd_times)
    # the separate calls of steps 1 and 2 (permute of Q, K, V; pool of Q, K), which the step
    # replaces by the fused call for Q and K: each timed on its own over a few iterations
    perm_times, pool_times = [], []
    for i in range(args.warmup + max(3, min(args.steps, 12))):
        a0, a1, a2 = event(), event(), event()
        a0.record(stream)
        V.permute_tiles(q, maps, bufs.q_t)
        V.permute_tiles(k, maps, bufs.k_t)
        V.permute_tiles(v, maps, bufs.v_t)
        a1.record(stream)
        V.tile_pool(bufs.q_t, maps, bufs.pooled_q)
        V.tile_pool(bufs.k_t, maps, bufs.pooled_k)
        a2.record(stream)
        a2.synchronize()
        if i >= args.warmup:
            perm_times.append(a0.elapsed_time(a1))
            pool_times.append(a1.elapsed_time(a2))
    V.check_device_status()
    perm_ms, pool_ms = statistics.median(perm_times), statistics.median(pool_times)
    attn_secondary = {
        "valid_token_tflops": valid_flop / (attn_ms * 1e-3) / 1e12,
        "executed_tflops": exec_flop / (attn_ms * 1e-3) / 1e12,
        "executed_frac_bf16_peak": exec_flop / (attn_ms * 1e-3) / 1e12 / peaks["bf16"],
        "executed_note": "tensor-core FLOP actually issued: key tiles with at most 64 valid slots are "
                         "computed over their first 64 keys",
        "dense_equivalent_tflops": 4.0 * D * N * N * H * B / (attn_ms * 1e-3) / 1e12,
        "random_lists_ms": rnd_ms,
        "random_lists_tflops": rnd_blocks * FLOP_PER_BLOCK / (rnd_ms * 1e-3) / 1e12,
        "random_lists_note": "fresh uniform lists (forced diagonal, same per-row budgets), 4 patterns cycled",
    }
    nbytes = N * H * D * 2
    hbm = {
        "permute_GBps": 3 * 2 * nbytes / (perm_ms * 1e-3) / 1e9,
        "pool_GBps": (2 * nbytes + 2 * w.nT * H * 3 * D * 4) / (pool_ms * 1e-3) / 1e9,
        "unpermute_GBps": 2 * nbytes / (stage_ms["unpermute"] * 1e-3) / 1e9,
        "permute_v_step_GBps": 2 * nbytes / (stage_ms["permute_v"] * 1e-3) / 1e9,
        "permute_pool_qk_fused_GBps": (2 * 2 * nbytes + 2 * w.nT * H * 3 * D * 4)
        / (stage_ms["permute_pool_qk"] * 1e-3) / 1e9,
    }
    for kname in list(hbm):
        hbm[kname.replace("_GBps", "_frac")] = hbm[kname] / peaks["hbm"]
    hbm["permute_pool_qk_fused_ms"] = stage_ms["permute_pool_qk"]
    hbm["permute_pool_qk_separate_ms"] = perm_ms * 2 / 3 + pool_ms
    hbm["separate_note"] = "permute and pool timed as separate calls after the timed steps"
    traffic = _attn_traffic(H)
    mhz = clk["sm_mhz"] if clk else 1965.0
    clock_peak = BF16_FLOP_PER_CLK_SM * 148 * mhz * 1e6 / 1e12

    line = {
        "metric": METRIC, "value": _job_tflops(world, flop_step, ms_step), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded smoothed-field Q/K, N(0,1) V, random-init projections)",
        "config": {"workload": f"clip16x9: B=1 H={H} grid 31x30x54 (50220 tokens) tile (1,8,16), "
                               "nT=496, density 1/10", "global_batch": world * B, "seq_len": N,
                   "parallelism": f"replicas x{world}", "visited_blocks": blocks,
                   "l2": f"inputs larger than L2 ({3 * N * H * D * 2 / 1e9:.2f} GB raster Q/K/V per step)"},
        "attn_ms_per_call": attn_ms, "attn_tflops": attn_tflops,
        "attn_frac_bf16_peak": attn_tflops / peaks["bf16"],
        "attn_frac_other_peaks": {"sustained": attn_tflops / peaks["bf16_sus"],
                                  "clock": attn_tflops / clock_peak, "clock_peak_tflops": clock_peak,
                                  "clock_note": "8192 FLOP/clk/SM x 148 SMs x median SM MHz sampled in the timed region"},
        "attn_secondary": attn_secondary,
        "stage_ms": stage_ms, "hbm_stages": hbm,
        "roofline": {"bound": "tensor", "achieved": attn_tflops, "peak": peaks["bf16"],
                     "unit": "TFLOP/s", "frac": attn_tflops / peaks["bf16"], "traffic": traffic,
                     "traffic_algorithmic": _attn_algorithmic_bytes(H, w.nT, B),
                     "kernel": "attn_fwd_kernel",
                     "peak_note": f"{peaks['source']} burst dense bf16 (the timed region lasts well under a "
                                  "second)"},
        "e2e": {"value": _job_tflops(world, flop_step, e_ms), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e_ms},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
    }
    if rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.cpu_seconds, inp)
    if rank == 0:
        print(json.dumps(line), flush=True)
    del bufs
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def workload(args) -> synth.Workload:
    """The 16:9-clip workload, or the same clip with fewer heads (--heads, for profiling)."""
    if args.heads == WORKLOAD.H:
        return WORKLOAD
    return synth.head_subset(WORKLOAD, list(range(args.heads)))


def _oracle_sample(inp, heads, rows_per_head):
    """The oracle's six steps on some heads of the workload, attention on some query tiles.

    Returns (visited-block FLOPs processed, seconds, seconds per step)."""
    from oracle import veda_oracle as O
    w = WORKLOAD
    t0 = time.perf_counter()
    marks = []
    f = lambda t: t[:, :, heads].double().numpy()
    q, k, v = f(inp.q), f(inp.k), f(inp.v)
    maps = [O.tile_map(w.grid, w.head_shapes[h], w.n_tail) for h in heads]
    slots, nv, seg = O.stack_maps(maps, w.nT)
    marks.append(time.perf_counter())
    qt, kt, vt = O.permute(q, slots), O.permute(k, slots), O.permute(v, slots)
    marks.append(time.perf_counter())
    pq, pk = O.pool(qt, nv), O.pool(kt, nv)
    marks.append(time.perf_counter())
    S = O.scores(pq, pk, inp.wq[heads].double().numpy(), inp.wk[heads].double().numpy())
    marks.append(time.perf_counter())
    lists = O.select(S, nv, seg, [len(m.n_valid) for m in maps], w.rho)
    marks.append(time.perf_counter())
    rows = [(0, j, r) for j in range(len(heads)) for r in range(rows_per_head)]
    o_t, _ = O.attention(qt, kt, vt, nv, lists, SCALE, rows=rows)
    marks.append(time.perf_counter())
    O.unpermute(np.nan_to_num(o_t), slots, w.N)
    marks.append(time.perf_counter())
    dt = marks[-1] - t0
    names = ["permute_qkv", "pool_qk", "scores", "select", "attention", "unpermute"]
    stage_s = {n: marks[i + 1] - marks[i] for i, n in enumerate(names)}
    blocks = sum(len(lists.full[0][j][r]) + len(lists.partial[0][j][r]) for (_, j, r) in rows)
    return blocks * FLOP_PER_BLOCK, dt, stage_s


def _cores():
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(seconds: float, inp):
    # whole path on heads 0.., attention on as many query tiles as fit the time budget
    # (calibrated: fixed cost of the non-attention steps + cost per attention query tile)
    _, t8, _ = _oracle_sample(inp, [0], 8)
    _, t24, _ = _oracle_sample(inp, [0], 24)
    per_row = max((t24 - t8) / 16, 1e-4)
    fixed = max(t8 - 8 * per_row, 0.0)
    heads = [0]
    rows = int((seconds - fixed) / per_row)
    while rows > WORKLOAD.nT * len(heads) and len(heads) < 4:
        heads.append(len(heads))
        rows = int((seconds - fixed * len(heads)) / per_row)
    rows = max(16, min(WORKLOAD.nT, rows // len(heads)))
    flop, dt, stage_s = _oracle_sample(inp, heads, rows)
    return {"value": flop / dt / 1e12, "unit": UNIT, "cores": _cores(), "kind": "oracle",
            "sample": f"fp64 oracle, all six steps on {len(heads)} of 40 heads, attention on {rows} of 496 "
                      f"query tiles per head ({dt:.1f} s); value = visited-block FLOPs / CPU time",
            "stage_s": stage_s}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    inp = synth.make_inputs(WORKLOAD)
    rows = args.ref_rows
    for _ in range(args.warmup):
        _oracle_sample(inp, [0], max(1, rows // 4))
    flops, secs = 0, 0.0
    stage_s = {}
    for _ in range(args.steps):
        f, dt, st = _oracle_sample(inp, [0], rows)
        flops += f
        secs += dt
        for n, x in st.items():
            stage_s[n] = stage_s.get(n, 0.0) + x / args.steps
    value = flops / secs / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (same seeded inputs as the CUDA arm)",
        "config": {"workload": "clip16x9: B=1 H=40 grid 31x30x54 (50220 tokens) tile (1,8,16), "
                               "nT=496, density 1/10", "global_batch": 1, "seq_len": WORKLOAD.N,
                   "parallelism": "cpu"},
        "cpu_baseline": {"kind": "oracle", "cores": _cores(), "value": value, "unit": UNIT,
                         "sample": f"each step: fp64 oracle, all six steps on head 0 of 40, "
                                   f"attention on {rows} of 496 query tiles", "stage_s": stage_s},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_heat(args):
    """Teacher block heat and mask quality on the 16:9 clip (not the contract line): the
    predicted path, every key tile listed (density 1/1), dense attention for the LSE, block
    heat over all blocks (timed), the oracle mask selected on the heat, and the attention mass
    kept by the predicted and by the oracle mask plus the predicted mask's recall. The heat
    kernel does one MUFU ex2 per score, so its roofline is the MUFU rate: 16 ex2 per cycle
    per SM x 148 SMs x the maximum SM clock."""
    from block_sparse_attention_max_b200 import veda as V
    dev = torch.device("cuda", torch.cuda.current_device())
    w = workload(args)
    inp = synth.make_inputs(w)
    maps = V.build_tile_map(w.grid, w.head_shapes, w.n_tail, inp.tile_order).to(dev)
    q, k, v, wq, wk = (t.to(dev) for t in (inp.q, inp.k, inp.v, inp.wq, inp.wk))
    bufs = V.sparse_attention(q, k, v, wq, wk, maps, w.rho, SCALE)
    B, H, Npad, D = bufs.q_t.shape
    nT = Npad // 128
    dense = V.select_blocks(torch.zeros((B, H, nT, nT), dtype=torch.float32, device=dev), maps,
                            [(1, 1)] * len(w.rho))
    blocks = _visited_blocks(dense)
    stream = torch.cuda.current_stream()

    def timed(fn, n):
        for _ in range(args.warmup):
            fn()
        times = []
        for _ in range(n):
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            fn()
            a1.record(stream)
            a1.synchronize()
            times.append(a0.elapsed_time(a1))
        return statistics.median(times)

    o_d = torch.empty_like(bufs.q_t)
    lse = torch.empty((B, H, Npad), dtype=torch.float32, device=dev)
    heat = torch.empty((B, H, nT, nT), dtype=torch.float32, device=dev)
    n = max(3, min(args.steps, 10))
    dense_ms = timed(lambda: V.block_sparse_attn_fwd(bufs.q_t, bufs.k_t, bufs.v_t, maps, dense, SCALE, o_d, lse), n)
    heat_ms = timed(lambda: V.block_heat(bufs.q_t, bufs.k_t, maps, dense, lse, SCALE, out=heat), n)
    orc = V.select_blocks(heat, maps, w.rho)
    q_pred = V.mask_quality(heat, maps, bufs.lists, orc)
    q_orc = V.mask_quality(heat, maps, orc, orc)
    V.check_device_status()
    ex2 = blocks * 128 * 128
    peak_ex2 = 16 * 148 * 1.965e9
    line = {
        "heat": f"clip16x9: B=1 H={H} grid 31x30x54 (50220 tokens) tile (1,8,16), nT={nT}, all blocks",
        "blocks": blocks, "dense_attn_ms": dense_ms,
        "dense_attn_tflops": blocks * FLOP_PER_BLOCK / (dense_ms * 1e-3) / 1e12,
        "heat_ms": heat_ms,
        "heat_roofline": {"bound": "alu", "achieved": ex2 / (heat_ms * 1e-3) / 1e12, "unit": "T ex2/s",
                          "peak": peak_ex2 / 1e12, "frac": ex2 / (heat_ms * 1e-3) / peak_ex2,
                          "peak_note": "MUFU: 16 ex2 per cycle per SM x 148 SMs x 1965 MHz (maximum SM clock)"},
        "heat_qk_tflops": blocks * 2 * 128 ** 3 / (heat_ms * 1e-3) / 1e12,
        "predicted_mask_mass": q_pred.mass, "oracle_mask_mass": q_orc.mass, "predicted_recall": q_pred.recall,
        "density": f"{w.rho[0][0]}/{w.rho[0][1]}",
    }
    print(json.dumps(line), flush=True)


def run_bwd(args):
    """Backward of the attention step on the 16:9 clip (not the contract line): the predicted
    path and forward, then the transposed lists and the backward (D, dQ, dK/dV) for a seeded
    output gradient, timed with CUDA events per stage. Algorithmic work: 2.5x the forward's
    4*128^3 FLOP per visited block (five 128^3 GEMMs); executed work: 14*128^3 (S and dP are
    recomputed in both kernels)."""
    from block_sparse_attention_max_b200 import veda as V
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks = _peaks()
    w = workload(args)
    inp = synth.make_inputs(w)
    maps = V.build_tile_map(w.grid, w.head_shapes, w.n_tail, inp.tile_order).to(dev)
    q, k, v, wq, wk = (t.to(dev) for t in (inp.q, inp.k, inp.v, inp.wq, inp.wk))
    bufs = V.sparse_attention(q, k, v, wq, wk, maps, w.rho, SCALE)
    gen = torch.Generator().manual_seed(1000 * w.wid + 8)
    do_t = V.permute_tiles(torch.randn(inp.q.shape, generator=gen).to(torch.bfloat16).to(dev), maps)
    blocks = _visited_blocks(bufs.lists)
    stream = torch.cuda.current_stream()
    t_ms, b_ms = [], []
    for i in range(args.warmup + max(3, min(args.steps, 10))):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        e[0].record(stream)
        tl = V.transpose_lists(bufs.lists, maps)
        e[1].record(stream)
        V.block_sparse_attn_bwd(bufs.q_t, bufs.k_t, bufs.v_t, bufs.o_t, do_t, bufs.lse, maps, bufs.lists, tl, SCALE)
        e[2].record(stream)
        e[2].synchronize()
        if i >= args.warmup:
            t_ms.append(e[0].elapsed_time(e[1]))
            b_ms.append(e[1].elapsed_time(e[2]))
    V.check_device_status()
    bms = statistics.median(b_ms)
    alg = blocks * 10 * 128 ** 3
    exe = blocks * 14 * 128 ** 3
    line = {
        "bwd": f"clip16x9: B=1 H={w.H} grid 31x30x54 (50220 tokens) tile (1,8,16), nT={w.nT}, density 1/10",
        "blocks": blocks, "transpose_lists_ms": statistics.median(t_ms), "bwd_ms": bms,
        "bwd_tflops_algorithmic": alg / (bms * 1e-3) / 1e12,
        "bwd_roofline": {"bound": "tensor", "achieved": alg / (bms * 1e-3) / 1e12, "unit": "TFLOP/s",
                         "peak": peaks["bf16"], "frac": alg / (bms * 1e-3) / 1e12 / peaks["bf16"],
                         "note": "algorithmic work (10*128^3 per block) against the measured burst bf16 peak",
                         "executed_tflops": exe / (bms * 1e-3) / 1e12,
                         "executed_frac": exe / (bms * 1e-3) / 1e12 / peaks["bf16"],
                         "executed_note": "MMA work the kernels issue (14*128^3 per block while S and dP are "
                                          "recomputed in both kernels)"},
    }
    print(json.dumps(line), flush=True)


def run_fp8(args):
    """FP8 variant of the attention step on the 16:9 clip (not the contract line): the
    predicted path, then e4m3 quantisation of the tiled Q, K and V (V with transposed tiles)
    and the FP8 attention over the same lists, timed with CUDA events (median of --steps calls
    after --warmup), beside the bf16 attention of the same lists. Roofline: 4*128^3 FLOP per
    visited block against twice the measured burst bf16 peak (the nominal fp8 / bf16
    ratio of the tensor cores); quantisation against the measured HBM copy rate on its
    algorithmic bytes (read 2 B and write 1 B per element of the three tensors)."""
    from block_sparse_attention_max_b200 import veda as V
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks = _peaks()
    w = workload(args)
    inp = synth.make_inputs(w)
    maps = V.build_tile_map(w.grid, w.head_shapes, w.n_tail, inp.tile_order).to(dev)
    q, k, v, wq, wk = (t.to(dev) for t in (inp.q, inp.k, inp.v, inp.wq, inp.wk))
    bufs = V.sparse_attention(q, k, v, wq, wk, maps, w.rho, SCALE)
    blocks = _visited_blocks(bufs.lists)
    stream = torch.cuda.current_stream()
    q8, sq = V.quantize_fp8(bufs.q_t)
    k8, sk = V.quantize_fp8(bufs.k_t)
    vt8, sv = V.quantize_fp8(bufs.v_t, transpose_tiles=True)
    o8 = torch.empty_like(bufs.o_t)
    lse8 = torch.empty_like(bufs.lse)
    ob = torch.empty_like(bufs.o_t)
    q_ms, a8_ms, ab_ms = [], [], []
    for i in range(args.warmup + args.steps):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        e[0].record(stream)
        V.quantize_fp8(bufs.q_t, codes=q8, scale=sq)
        V.quantize_fp8(bufs.k_t, codes=k8, scale=sk)
        V.quantize_fp8(bufs.v_t, transpose_tiles=True, codes=vt8, scale=sv)
        e[1].record(stream)
        V.block_sparse_attn_fwd_fp8(q8, k8, vt8, sq, sk, sv, maps, bufs.lists, SCALE, out=o8, lse=lse8)
        e[2].record(stream)
        V.block_sparse_attn_fwd(bufs.q_t, bufs.k_t, bufs.v_t, maps, bufs.lists, SCALE, out=ob, lse=bufs.lse)
        e[3].record(stream)
        e[3].synchronize()
        if i >= args.warmup:
            q_ms.append(e[0].elapsed_time(e[1]))
            a8_ms.append(e[1].elapsed_time(e[2]))
            ab_ms.append(e[2].elapsed_time(e[3]))
    V.check_device_status()
    qms, ams, bms = statistics.median(q_ms), statistics.median(a8_ms), statistics.median(ab_ms)
    flop = blocks * 4 * 128 ** 3
    elems = 3 * bufs.q_t.numel()
    d = (o8.float() - ob.float()).abs()
    line = {
        "fp8": f"clip16x9: B=1 H={w.H} grid 31x30x54 (50220 tokens) tile (1,8,16), nT={w.nT}, density 1/10",
        "blocks": blocks, "quantize_qkv_ms": qms,
        "quantize_GBps": elems * 3 / (qms * 1e-3) / 1e9,
        "quantize_frac_hbm": elems * 3 / (qms * 1e-3) / 1e9 / peaks["hbm"],
        "attn_fp8_ms": ams, "attn_fp8_tflops": flop / (ams * 1e-3) / 1e12,
        "attn_bf16_ms": bms, "attn_bf16_tflops": flop / (bms * 1e-3) / 1e12,
        "fp8_roofline": {"bound": "tensor", "achieved": flop / (ams * 1e-3) / 1e12, "unit": "TFLOP/s",
                         "peak": 2 * peaks["bf16"], "frac": flop / (ams * 1e-3) / 1e12 / (2 * peaks["bf16"]),
                         "peak_note": "measured burst bf16 x 2 (nominal fp8 / bf16 ratio)"},
        "fp8_vs_bf16_output": {"max_abs": float(d.max()), "mean_abs": float(d.mean()),
                               "mean_abs_bf16_output": float(ob.float().abs().mean())},
    }
    print(json.dumps(line), flush=True)


PLAN_CANDIDATES = [(1, 8, 16), (2, 8, 8), (4, 4, 8), (2, 4, 16), (1, 16, 8)]


def run_plan(args):
    """Oracle tile-plan search on the 16:9 clip (not the contract line): for each candidate
    tile shape, permute, dense attention for the LSE, block heat, oracle mask, sparse
    attention and relative output error per head, then the vote (at most two shapes)."""
    from block_sparse_attention_max_b200 import plan
    dev = torch.device("cuda", torch.cuda.current_device())
    w = workload(args)
    inp = synth.make_inputs(w)
    q, k, v = (t.to(dev) for t in (inp.q, inp.k, inp.v))
    plan.tile_plan_search(q, k, v, w.grid, w.n_tail, PLAN_CANDIDATES[:1], w.rho, SCALE)   # warm-up
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record()
    res = plan.tile_plan_search(q, k, v, w.grid, w.n_tail, PLAN_CANDIDATES, w.rho, SCALE)
    ev1.record()
    torch.cuda.synchronize()
    line = {
        "plan": f"clip16x9: B=1 H={w.H} grid 31x30x54 (50220 tokens), density 1/10, "
                f"{len(PLAN_CANDIDATES)} candidate shapes",
        "search_ms_gpu": ev0.elapsed_time(ev1), "search_s_wall": time.perf_counter() - t0,
        "mean_error_per_shape": {f"{t}x{h}x{ww}": float(res.errors[:, c].mean())
                                 for c, (t, h, ww) in enumerate(PLAN_CANDIDATES)},
        "kept_shapes": [f"{t}x{h}x{ww}" for (t, h, ww) in (PLAN_CANDIDATES[c] for c in res.kept)],
        "heads_per_kept_shape": {f"{t}x{h}x{ww}": int((res.assign == c).sum())
                                 for c, (t, h, ww) in ((c, PLAN_CANDIDATES[c]) for c in res.kept)},
    }
    print(json.dumps(line), flush=True)


def run_sweep(args):
    """Density and length sweep of the attention step (not the contract line): for each
    configuration, permute/pool/score/select once, then time the attention call alone
    (CUDA events, median of --steps calls after --warmup). Writes one JSON line per
    configuration; at 100% density the same kernel runs dense attention."""
    from block_sparse_attention_max_b200 import veda as V
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks = _peaks()
    cfgs = [synth.sweep_density(p, q) for p, q in synth.SWEEP_DENSITIES]
    cfgs += [synth.sweep_length(T) for T in synth.SWEEP_FRAMES]
    cache = {}
    for w in cfgs:
        key = (w.grid, w.wid)
        if key not in cache:                 # the density configs share one set of inputs
            cache.clear()
            cache[key] = synth.make_inputs(w)
        inp = cache[key]
        maps = V.build_tile_map(w.grid, w.head_shapes, w.n_tail, inp.tile_order).to(dev)
        q, k, v = (t.to(dev) for t in (inp.q, inp.k, inp.v))
        B, N, H, D = q.shape
        bufs = V.sparse_attention(q, k, v, inp.wq.to(dev), inp.wk.to(dev), maps, w.rho, SCALE)
        V.check_device_status()
        blocks = _visited_blocks(bufs.lists)
        times = []
        for it in range(args.warmup + args.steps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            V.block_sparse_attn_fwd(bufs.q_t, bufs.k_t, bufs.v_t, maps, bufs.lists, SCALE, bufs.o_t, bufs.lse)
            e1.record()
            torch.cuda.synchronize()
            if it >= args.warmup:
                times.append(e0.elapsed_time(e1))
        V.check_device_status()
        ms = statistics.median(times)
        tf = blocks * FLOP_PER_BLOCK / (ms * 1e-3) / 1e12
        print(json.dumps({"sweep": w.name, "tokens": N, "nT": maps.nT, "density": f"{w.rho[0][0]}/{w.rho[0][1]}",
                          "visited_blocks": blocks, "attn_ms": ms, "attn_tflops": tf,
                          "frac_bf16_peak_burst": tf / peaks["bf16"]}), flush=True)
        del bufs, q, k, v
        torch.cuda.empty_cache()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["veda", "reference"], default="veda")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--clocks-csv", default=None,
                    help="where to keep the nvidia-smi samples of the timed region (default: a temp file)")
    ap.add_argument("--ref-rows", type=int, default=24)
    ap.add_argument("--plan", action="store_true",
                    help="oracle tile-plan search on the clip (one JSON line)")
    ap.add_argument("--bwd", action="store_true",
                    help="backward of the attention step on the clip (one JSON line)")
    ap.add_argument("--heat", action="store_true",
                    help="teacher block heat and mask quality on the clip (one JSON line)")
    ap.add_argument("--fp8", action="store_true",
                    help="FP8 (e4m3) variant of the attention step on the clip (one JSON line)")
    ap.add_argument("--sweep", action="store_true",
                    help="density / length sweep of the attention step (one JSON line per config)")
    ap.add_argument("--heads", type=int, default=WORKLOAD.H,
                    help="heads of the 16:9 clip to run (default all 40; fewer for profiling)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "veda":
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    elif args.sweep:
        run_sweep(args)
    elif args.fp8:
        run_fp8(args)
    elif args.heat:
        run_heat(args)
    elif args.bwd:
        run_bwd(args)
    elif args.plan:
        run_plan(args)
    else:
        run_veda(args)


if __name__ == "__main__":
    main()
