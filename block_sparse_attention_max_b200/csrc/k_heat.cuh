// k_heat.cuh -- teacher block heat from the dense LSE, and the quality of a block mask.
//
// "Miowtion" README, Key Features / Veda sparse attention: the predictor learns from teacher
// block heat computed from the dense LSE. heat[b, h, i, j] = mean over the valid query slots
// q of tile i of the sum over the valid key slots k of tile j of exp(scale q.k - LSE_q), with
// LSE_q the log-sum-exp of dense attention (the forward kernel's LSE output at full density).
// "Deploying this checkpoint" sections 4 and 6: the predictor is judged by its recall against
// the oracle mask, and by the attention mass a mask keeps (an oracle mask keeps ~0.63 of it
// at a 10% keep ratio).
//
// heat_kernel runs the forward kernel's Q K^T stream (same producer, same issuer, same
// double-buffered S in tensor memory) over the listed blocks -- all of them for dense heat --
// and replaces softmax + P V with exact probabilities against the given LSE: the eight warps
// each sum their 16 rows of one block and add the sum into heat[b, h, i, j]. It does half the
// forward's tensor work and the same MUFU work (one ex2 per score).
#pragma once

#include "k_attn.cuh"

namespace veda {
namespace heat {

struct HeatArgs {
  attn::Args a;        // lists, tile_valid, items, H, nT, stride (o / lse / scale unused)
  const float* lse;    // [B*H*nT*128] natural-log LSE of dense attention
  float* heat;         // [B*H*nT][nT]; zeroed by the host, blocks add into it
  float scale_log2;    // softmax scale * log2(e)
};

constexpr uint32_t kTmemCols = 256;   // S0 | S1
constexpr float kLog2e = 1.4426950408889634f;

// Loads S of blocks g .. g + NB - 1 (handing each TMEM buffer back as soon as it is in
// registers), then computes their probabilities in one loop, so the exponentials of the NB
// blocks run back to back and the per-block waits, hand-backs and reductions are paid once
// per group. A thread holds rows r0 and r0 + 8 and 32 scores of each per block (16x256b
// shape, as in the forward kernel). Returns false when a wait gave up.
template <int NB>
__device__ __forceinline__ bool heat_group(attn::Bars& bars, uint32_t tmem, uint32_t lane_off, uint32_t c,
                                           uint32_t lane, uint32_t g, uint64_t c2, uint64_t nlx0, uint64_t nlx1,
                                           float inv_nq, float* heat_row, volatile int* abort) {
  using namespace attn;
  uint32_t s[NB][64];
  int32_t key[NB];
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    const uint32_t gb = g + b, sbuf = gb & 1;
    if (!warp_wait_abort(smem_u32(&bars.rec_full[gb % kRec]), (gb / kRec) & 1, abort, 36)) return false;
    const int32_t nv = reinterpret_cast<volatile int32_t*>(bars.rec_nv)[gb % kRec];
    key[b] = reinterpret_cast<volatile int32_t*>(bars.rec_idx)[gb % kRec];
    if (!warp_wait_abort(smem_u32(&bars.s_full[sbuf]), (gb >> 1) & 1, abort, 30)) return false;
    tc_fence_after();
    tmem_ld_16x256b_x16(tmem + lane_off + kColS + sbuf * 128, s[b]);
    tmem_wait_ld();
    reg_fence(s[b]);
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&bars.s_free[sbuf]));
    if (nv < 128) {
      // column 8k + 2c + e is a key slot < nv exactly for k < ceil((nv - 2c - e) / 8)
      const int32_t kv0 = (nv - 2 * static_cast<int32_t>(c) + 7) >> 3;
      const int32_t kv1 = (nv - 2 * static_cast<int32_t>(c) + 6) >> 3;
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        if (k >= kv0) { s[b][4 * k] = 0xFF800000u; s[b][4 * k + 2] = 0xFF800000u; }   // -inf
        if (k >= kv1) { s[b][4 * k + 1] = 0xFF800000u; s[b][4 * k + 3] = 0xFF800000u; }
      }
    }
  }
  uint64_t acc[NB][2];
#pragma unroll
  for (int b = 0; b < NB; ++b) acc[b][0] = acc[b][1] = 0ull;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      float x0, x1, y0, y1;
      f2_unpack(f2_fma(f2_pack(s[b][4 * k], s[b][4 * k + 1]), c2, nlx0), x0, x1);
      const uint64_t yy = f2_fma(f2_pack(s[b][4 * k + 2], s[b][4 * k + 3]), c2, nlx1);
      const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
      float q0, q1;
      if ((k & 3) == 3) {
        exp2_fma_x2(yy, q0, q1);   // an eighth of the exponentials on the FMA pipe
      } else {
        f2_unpack(yy, y0, y1);
        q0 = ex2_approx(y0);
        q1 = ex2_approx(y1);
      }
      acc[b][k & 1] = f2_add(acc[b][k & 1], f2_add(f2_pack(__float_as_uint(p0), __float_as_uint(p1)),
                                                   f2_pack(__float_as_uint(q0), __float_as_uint(q1))));
    }
  }
  float t[NB];
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    float t0, t1, t2, t3;
    f2_unpack(acc[b][0], t0, t1);
    f2_unpack(acc[b][1], t2, t3);
    t[b] = (t0 + t1) + (t2 + t3);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
    for (int b = 0; b < NB; ++b) t[b] += __shfl_xor_sync(0xffffffffu, t[b], o);
  }
  if (lane == 0) {
#pragma unroll
    for (int b = 0; b < NB; ++b) atomicAdd(heat_row + key[b], t[b] * inv_nq);
  }
  return true;
}

// The eight softmax warps: warp w owns tile rows 32 (w % 4) + 16 (w / 4) + [0, 16) of every
// block and takes an item's blocks two at a time (the last one alone when the item has an odd
// count).
__device__ __forceinline__ void heat_softmax(const HeatArgs& p, attn::Bars& bars, uint32_t tmem, uint32_t warp,
                                             uint32_t lane) {
  using namespace attn;
  const Args& a = p.a;
  volatile int* abort = &bars.abort;
  const uint32_t base = 32 * (warp & 3) + 16 * (warp >> 2);
  const uint32_t lane_off = base << 16;
  const uint32_t r0 = base + lane / 4, c = lane & 3;
  const uint64_t c2 = f2_pack(__float_as_uint(p.scale_log2), __float_as_uint(p.scale_log2));
  uint32_t g = 0;
  for (int64_t mm = 0;; ++mm) {
    const int64_t u = cta_item(mm);
    if (u >= a.items) break;
    int32_t nf;
    bool bad;
    const int32_t n = item_blocks(a, u, nf, bad);
    if (n == 0) {
      if (bad && lane == 0 && warp == 0) flag_status(ST_BAD_LIST);
      continue;
    }
    const int32_t h = static_cast<int32_t>((u / a.nT) % a.H), i = static_cast<int32_t>(u % a.nT);
    int32_t nq = a.valid[static_cast<int64_t>(h) * a.nT + i];
    nq = nq < 0 ? 0 : (nq > 128 ? 128 : nq);
    // -LSE in log2 units per row; pad query slots get -inf, so their probabilities are 0
    const float nl0 = static_cast<int32_t>(r0) < nq ? -p.lse[u * 128 + r0] * kLog2e : -INFINITY;
    const float nl1 = static_cast<int32_t>(r0 + 8) < nq ? -p.lse[u * 128 + r0 + 8] * kLog2e : -INFINITY;
    const uint64_t nlx0 = f2_pack(__float_as_uint(nl0), __float_as_uint(nl0));
    const uint64_t nlx1 = f2_pack(__float_as_uint(nl1), __float_as_uint(nl1));
    const float inv_nq = nq > 0 ? 1.0f / static_cast<float>(nq) : 0.f;
    float* heat_row = p.heat + u * a.nT;
    bool ok = true;
    int32_t j = 0;
    for (; j + 2 <= n; j += 2, g += 2)
      if (!heat_group<2>(bars, tmem, lane_off, c, lane, g, c2, nlx0, nlx1, inv_nq, heat_row, abort)) { ok = false; break; }
    if (ok && j < n) {
      ok = heat_group<1>(bars, tmem, lane_off, c, lane, g, c2, nlx0, nlx1, inv_nq, heat_row, abort);
      ++g;
    }
    if (!ok) break;
  }
}

__global__ void __launch_bounds__(attn::kThreads, 1)
heat_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK, const HeatArgs p) {
  using namespace attn;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ Bars bars;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const uint32_t tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, wg = warp >> 2;
  volatile int* abort = &bars.abort;

  if (tid == 0) init_bars(bars);
  if (warp == 9) {
    tmem_alloc(smem_u32(&bars.tmem_base), kTmemCols);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    prefetch_tensormap(&tmQ);
    prefetch_tensormap(&tmK);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;

  if (wg == 2) {
    reg_dealloc<kControlRegs>();
    if (warp == 8 && lane == 0)
      role_qk_producer<false>(p.a, bars, sb, &tmQ, &tmK, abort);
    else if (warp == 9 && lane == 0)
      role_qk_issuer(bars, sb, tmem, abort);
  } else {
    reg_alloc<kSoftmaxRegs>();
    heat_softmax(p, bars, tmem, warp, lane);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9) tmem_dealloc(tmem, kTmemCols);
}

// ------------------------------------------------------------------------------------
// Mask quality: one warp per (b, h, query tile) row. The oracle list's tiles are marked in a
// per-warp bitmap; the predicted list's tiles then add their heat (kept mass) and count the
// marked ones (hits). Row results go to mass_rows / recall_rows; totals[4] accumulate
// (sum of n_valid * mass, sum of n_valid, sum of recall, rows with an oracle list).
// ------------------------------------------------------------------------------------
constexpr int kQualWarps = 4;
constexpr int kQualMaxTiles = 2048;

struct QualityArgs {
  const float* heat;            // [B*H*nT][nT]
  const int32_t* valid;         // [H][nT]
  const int32_t* nT_per_head;   // [H]
  const int32_t *pfc, *pfi, *ppc, *ppi;   // predicted lists
  const int32_t *ofc, *ofi, *opc, *opi;   // oracle lists
  int32_t pstride, ostride;
  float* mass_rows;             // [B*H*nT]
  float* recall_rows;           // [B*H*nT]
  float* totals;                // [4], zeroed by the host
  int32_t H, nT;
  int64_t rows;                 // B*H*nT
};

__device__ __forceinline__ int32_t list_entry(const int32_t* fi, const int32_t* pi, int64_t u, int32_t stride,
                                              int32_t nf, int32_t e) {
  return e < nf ? fi[u * stride + e] : pi[u * stride + (e - nf)];
}

__global__ void __launch_bounds__(32 * kQualWarps) mask_quality_kernel(const QualityArgs q) {
  __shared__ uint32_t bits[kQualWarps][kQualMaxTiles / 32];
  const uint32_t w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t u = static_cast<int64_t>(blockIdx.x) * kQualWarps + w;
  if (u >= q.rows) return;
  const int32_t i = static_cast<int32_t>(u % q.nT), h = static_cast<int32_t>((u / q.nT) % q.H);
  const int32_t nth = q.nT_per_head[h];
  if (nth < 0 || nth > q.nT) {
    if (lane == 0) flag_status(ST_BAD_LIST);
    return;
  }
  if (i >= nth) {
    if (lane == 0) { q.mass_rows[u] = 0.f; q.recall_rows[u] = 0.f; }
    return;
  }
  const int32_t pnf = q.pfc[u], pnp = q.ppc[u], onf = q.ofc[u], onp = q.opc[u];
  const bool bad = pnf < 0 || pnp < 0 || onf < 0 || onp < 0 || pnf > q.pstride || pnp > q.pstride ||
                   onf > q.ostride || onp > q.ostride;
  if (bad) {
    if (lane == 0) { flag_status(ST_BAD_LIST); q.mass_rows[u] = 0.f; q.recall_rows[u] = 0.f; }
    return;
  }
  uint32_t* bw = bits[w];
  for (int32_t x = static_cast<int32_t>(lane); x < kQualMaxTiles / 32; x += 32) bw[x] = 0u;
  __syncwarp();
  int32_t badidx = 0;
  for (int32_t e = static_cast<int32_t>(lane); e < onf + onp; e += 32) {
    const int32_t j = list_entry(q.ofi, q.opi, u, q.ostride, onf, e);
    if (j < 0 || j >= nth) { badidx = 1; continue; }
    atomicOr(&bw[j >> 5], 1u << (j & 31));
  }
  __syncwarp();
  float mass = 0.f;
  int32_t hits = 0;
  const float* hrow = q.heat + u * q.nT;
  for (int32_t e = static_cast<int32_t>(lane); e < pnf + pnp; e += 32) {
    const int32_t j = list_entry(q.pfi, q.ppi, u, q.pstride, pnf, e);
    if (j < 0 || j >= nth) { badidx = 1; continue; }
    mass += hrow[j];
    hits += (bw[j >> 5] >> (j & 31)) & 1u;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mass += __shfl_xor_sync(0xffffffffu, mass, o);
    hits += __shfl_xor_sync(0xffffffffu, hits, o);
    badidx |= __shfl_xor_sync(0xffffffffu, badidx, o);
  }
  if (lane == 0) {
    if (badidx) flag_status(ST_BAD_LIST);
    const int32_t ocount = onf + onp;
    const float recall = ocount > 0 ? static_cast<float>(hits) / static_cast<float>(ocount) : 0.f;
    q.mass_rows[u] = mass;
    q.recall_rows[u] = recall;
    const float wgt = static_cast<float>(q.valid[static_cast<int64_t>(h) * q.nT + i]);
    atomicAdd(q.totals + 0, wgt * mass);
    atomicAdd(q.totals + 1, wgt);
    if (ocount > 0) {
      atomicAdd(q.totals + 2, recall);
      atomicAdd(q.totals + 3, 1.0f);
    }
  }
}

// ------------------------------------------------------------------------------------
// Relative output error per head (the tile-plan search's criterion): sums over all tokens of
// |o - o_ref|^2 and |o_ref|^2 per head, raster [B][N][H][128] bf16. 16 threads per 256-byte
// row; per-CTA partial sums in shared memory, one atomic pair per CTA and head.
// ------------------------------------------------------------------------------------
constexpr int kErrThreads = 256;
constexpr int kErrMaxHeads = 256;

__global__ void __launch_bounds__(kErrThreads) rel_error_kernel(const __nv_bfloat16* __restrict__ o,
                                                                const __nv_bfloat16* __restrict__ ref,
                                                                float* __restrict__ sums, int64_t rows, int32_t H) {
  __shared__ float part[kErrMaxHeads][2];
  for (int i = threadIdx.x; i < H * 2; i += blockDim.x) (&part[0][0])[i] = 0.f;
  __syncthreads();
  const uint32_t c = threadIdx.x & 15;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * (kErrThreads / 16);
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * (kErrThreads / 16) + (threadIdx.x >> 4); r < rows; r += stride) {
    const uint4 x = *reinterpret_cast<const uint4*>(o + r * 128 + c * 8);
    const uint4 y = *reinterpret_cast<const uint4*>(ref + r * 128 + c * 8);
    const __nv_bfloat162* xp = reinterpret_cast<const __nv_bfloat162*>(&x);
    const __nv_bfloat162* yp = reinterpret_cast<const __nv_bfloat162*>(&y);
    float e = 0.f, n = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 a2 = __bfloat1622float2(xp[i]), b2 = __bfloat1622float2(yp[i]);
      const float d0 = a2.x - b2.x, d1 = a2.y - b2.y;
      e = fmaf(d0, d0, fmaf(d1, d1, e));
      n = fmaf(b2.x, b2.x, fmaf(b2.y, b2.y, n));
    }
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) {
      e += __shfl_xor_sync(0xffffffffu, e, off);
      n += __shfl_xor_sync(0xffffffffu, n, off);
    }
    if (c == 0) {
      const int32_t h = static_cast<int32_t>(r % H);
      atomicAdd(&part[h][0], e);
      atomicAdd(&part[h][1], n);
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < H; i += blockDim.x) {
    atomicAdd(sums + 2 * i, part[i][0]);
    atomicAdd(sums + 2 * i + 1, part[i][1]);
  }
}

}  // namespace heat
}  // namespace veda
