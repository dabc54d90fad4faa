// k_fp8.cuh -- FP8 (e4m3) variant of step 5: quantisation of the tiled Q / K / V and the
// block-sparse attention forward with e4m3 operands on the tensor cores.
//
// The pages ship their predictor in FP8 ("Deploying this checkpoint", preamble and section
// 3) but give no FP8 attention; this variant follows the same steps as the bf16 kernel
// (k_attn.cuh) over the same block lists, with:
//   * one scale per (batch, head) tensor: scale = amax / 448, code = e4m3(x * 448 / amax),
//     both in fp32, rounding to nearest even and saturating at +-448 (cvt.rn.satfinite);
//     V is stored as transposed tiles ([channel][key position]) so that both products take
//     K-major operands, with the keys of every group of 16 in the order the softmax packs P
//     (position 16m + 4c + e holds key slot 16m + 2c + (e & 1) + 8 (e >> 1));
//   * S = Q K^T from e4m3 operands (kind::f8f6f4, K = 32 per MMA), scaled by
//     q_scale * k_scale * softmax_scale in the softmax;
//   * every role visits an item's diagonal key tile first (it holds most rows' maxima), then
//     the rest of the list in order;
//   * P = 2^(s - m + 7) in e4m3 (the reference m moves when a row maximum grows by more
//     than 1.75, so P stays below 2^8.75 = 430 < 448), written by the softmax warps into
//     tensor memory (four keys per 32-bit column, in the order above); O += P V with P read
//     from tensor memory and V from its transposed tile, O = O_acc * v_scale / l in the
//     epilogue.
// Roles, rings, barriers and bounded waits are those of the bf16 kernel (attn::Bars).
#pragma once

#include "k_attn.cuh"

namespace veda {
namespace fp8 {

// ---------------------------------------------------------------- quantisation
constexpr int kQuantThreads = 256;
constexpr int64_t kAmaxChunk = 32768;    // bf16 elements per amax work unit
constexpr float kE4m3Max = 448.0f;

struct QuantArgs {
  const __nv_bfloat16* x;     // [BH][rows][128] bf16
  uint8_t* codes;             // [BH][rows][128] e4m3
  uint32_t* amax_bits;        // [BH]: fp32 bits of max |x| (the caller's scale buffer, zeroed)
  float* scale;               // [BH]: amax / 448 (written last, over amax_bits)
  int64_t bh;                 // B * H
  int64_t rows;               // nT * 128 rows per (b, h)
  int32_t transpose;          // store every 128 x 128 tile transposed
};

// max |x| per (b, h): CTAs take 32768-element chunks; non-negative floats order as integers
__global__ void __launch_bounds__(kQuantThreads) amax_kernel(const QuantArgs q) {
  __shared__ float red[kQuantThreads / 32];
  const int64_t per_bh = q.rows * 128;
  const int64_t chunks = (per_bh + kAmaxChunk - 1) / kAmaxChunk;
  const int64_t units = q.bh * chunks;
  for (int64_t u = blockIdx.x; u < units; u += gridDim.x) {
    const int64_t b = u / chunks, ch = u % chunks;
    const int64_t beg = ch * kAmaxChunk;
    const int64_t end = per_bh < beg + kAmaxChunk ? per_bh : beg + kAmaxChunk;
    const uint4* src = reinterpret_cast<const uint4*>(q.x + b * per_bh);
    float m = 0.f;
    auto fold = [&](const uint4& v) {
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        m = fmaxf(m, __uint_as_float((w[k] << 16) & 0x7fffffffu));   // |low bf16| as fp32
        m = fmaxf(m, __uint_as_float(w[k] & 0x7fff0000u));           // |high bf16|
      }
    };
    int64_t i = beg / 8 + threadIdx.x;
    // eight independent 16-byte loads in flight per thread, then the remainder
    for (; i + 7 * kQuantThreads < end / 8; i += 8 * kQuantThreads) {
      uint4 v[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) v[k] = src[i + k * kQuantThreads];
#pragma unroll
      for (int k = 0; k < 8; ++k) fold(v[k]);
    }
    for (; i < end / 8; i += kQuantThreads) fold(src[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
      float t = red[0];
      for (int i = 1; i < kQuantThreads / 32; ++i) t = fmaxf(t, red[i]);
      atomicMax(q.amax_bits + b, __float_as_uint(t));
    }
    __syncthreads();
  }
}

// e4m3 codes of one 128 x 128 tile per CTA iteration: thread (row r, half) converts 64
// elements; with transpose the codes go through shared memory and leave as [channel][key
// position], position 16m + 4c + e of a row holding key slot 16m + 2c + (e & 1) + 8 (e >> 1)
// (the order in which the attention's softmax packs P into tensor memory).
// (kQuantThreads = 256: 128 rows x 2 halves, and 32 channel groups x 8 key groups.)
__global__ void __launch_bounds__(kQuantThreads) quant_kernel(const QuantArgs q) {
  __shared__ __align__(16) uint8_t tile[128][144];
  const int64_t tiles_per_bh = q.rows / 128;
  const int64_t tiles = q.bh * tiles_per_bh;
  const int r = static_cast<int>(threadIdx.x >> 1), half = static_cast<int>(threadIdx.x & 1);
  for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x) {
    const float amax = __uint_as_float(q.amax_bits[t / tiles_per_bh]);
    const float inv = amax > 0.f ? __fdiv_rn(kE4m3Max, amax) : 1.0f;
    const uint4* src = reinterpret_cast<const uint4*>(q.x + (t * 128 + r) * 128 + half * 64);
    uint32_t out[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint4 v = src[i];
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; k += 2) {
        const float f0 = __uint_as_float(w[k] << 16), f1 = __uint_as_float(w[k] & 0xffff0000u);
        const float f2 = __uint_as_float(w[k + 1] << 16), f3 = __uint_as_float(w[k + 1] & 0xffff0000u);
        const uint32_t lo = pack_e4m3x2(__fmul_rn(f0, inv), __fmul_rn(f1, inv));
        const uint32_t hi = pack_e4m3x2(__fmul_rn(f2, inv), __fmul_rn(f3, inv));
        out[2 * i + k / 2] = lo | (hi << 16);
      }
    }
    if (!q.transpose) {
      uint4* dst = reinterpret_cast<uint4*>(q.codes + (t * 128 + r) * 128 + half * 64);
#pragma unroll
      for (int i = 0; i < 4; ++i) dst[i] = make_uint4(out[4 * i], out[4 * i + 1], out[4 * i + 2], out[4 * i + 3]);
    } else {
      uint32_t* row = reinterpret_cast<uint32_t*>(&tile[r][half * 64]);
#pragma unroll
      for (int i = 0; i < 16; ++i) row[i] = out[i];
      __syncthreads();
      // thread (channel group cg, key group kg): channels 4 cg .. + 3 of key slots 16 kg .. + 15,
      // read as 32-bit words (consecutive words across the warp) and transposed 4 x 4 bytes at
      // a time in registers; output rows are channels, 16 key bytes each, word i of a group
      // holding key slots 2i, 2i + 1, 2i + 8, 2i + 9 of it
      const int cg = static_cast<int>(threadIdx.x & 31), kg = static_cast<int>(threadIdx.x >> 5);
      uint32_t o[4][4];   // o[channel j][key word i]
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int k0 = 16 * kg + 2 * i;
        const uint32_t a0 = *reinterpret_cast<const uint32_t*>(&tile[k0][4 * cg]);
        const uint32_t a1 = *reinterpret_cast<const uint32_t*>(&tile[k0 + 1][4 * cg]);
        const uint32_t a2 = *reinterpret_cast<const uint32_t*>(&tile[k0 + 8][4 * cg]);
        const uint32_t a3 = *reinterpret_cast<const uint32_t*>(&tile[k0 + 9][4 * cg]);
        const uint32_t t0 = __byte_perm(a0, a1, 0x5140), t1 = __byte_perm(a2, a3, 0x5140);
        const uint32_t t2 = __byte_perm(a0, a1, 0x7362), t3 = __byte_perm(a2, a3, 0x7362);
        o[0][i] = __byte_perm(t0, t1, 0x5410);   // channel 4 cg: keys k0, k0 + 1, k0 + 8, k0 + 9
        o[1][i] = __byte_perm(t0, t1, 0x7632);
        o[2][i] = __byte_perm(t2, t3, 0x5410);
        o[3][i] = __byte_perm(t2, t3, 0x7632);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j)
        *reinterpret_cast<uint4*>(q.codes + (t * 128 + 4 * cg + j) * 128 + 16 * kg) =
            make_uint4(o[j][0], o[j][1], o[j][2], o[j][3]);
      __syncthreads();
    }
  }
}

// amax bits -> scale, in place, after the codes are written (stream order)
__global__ void scale_kernel(uint32_t* amax_bits, int64_t bh) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < bh) {
    const float a = __uint_as_float(amax_bits[i]);
    const float s = a > 0.f ? __fdiv_rn(a, kE4m3Max) : 1.0f;
    amax_bits[i] = __float_as_uint(s);
  }
}

// ---------------------------------------------------------------- attention
using attn::Bars;
using attn::cta_item;
using attn::item_blocks;
using attn::item_key;
using attn::opaque;
using attn::warp_wait_abort;
using attn::kOpFirstItem;
using attn::kOpLastBlk;
using attn::kOpNewItem;
using attn::kOpQBufShift;
using attn::kOpStop;
using attn::kQSt;
using attn::kKSt;
using attn::kVSt;
using attn::kRec;

// Position of the diagonal key tile (the query tile's own index) in an item's list, or -1.
// The full and the partial lists are ascending, so each takes one binary search; every role
// calls this, so all of them visit the blocks in the same order.
__device__ __forceinline__ int32_t diag_pos(const attn::Args& a, int64_t u, int32_t nf, int32_t n) {
  const int32_t i = static_cast<int32_t>(u % a.nT);
  const int32_t* f = a.full_idx + u * a.stride;
  int32_t lo = 0, hi = nf;
  while (lo < hi) {
    const int32_t mid = (lo + hi) >> 1;
    if (f[mid] < i) lo = mid + 1; else hi = mid;
  }
  if (lo < nf && f[lo] == i) return lo;
  const int32_t* pp = a.part_idx + u * a.stride;
  const int32_t np = n - nf;
  lo = 0;
  hi = np;
  while (lo < hi) {
    const int32_t mid = (lo + hi) >> 1;
    if (pp[mid] < i) lo = mid + 1; else hi = mid;
  }
  return (lo < np && pp[lo] == i) ? nf + lo : -1;
}
// List position visited at step j: the diagonal first, then the others in list order.
__device__ __forceinline__ int32_t visit_pos(int32_t j, int32_t d) {
  return d < 0 ? j : (j == 0 ? d : (j <= d ? j - 1 : j));
}

constexpr int kThreads = 384;
constexpr uint32_t kTileB = 16384;                             // 128 x 128 e4m3
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kQSt * kTileB;
constexpr uint32_t kOffV = kOffK + kKSt * kTileB;              // V tiles transposed
constexpr uint32_t kSmemTiles = kOffV + kVSt * kTileB;         // 112 KB
constexpr uint32_t kSmemBytes = kSmemTiles + 1024;             // + alignment slack
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256, kColP = 384;        // S0 | S1 | O | P0 | P1 (32 columns each)
constexpr uint32_t kIdesc = idesc_e4m3_f32(128, 128);
constexpr float kPExp = 7.0f;                                  // P as e4m3 of 2^7 p
constexpr float kRescaleLog2 = 1.75f;                          // 2^(7 + 1.75) = 430 < 448
constexpr float kLn2 = 0.69314718055994531f;

struct Args {
  attn::Args a;                 // lists, tile_valid, o, lse, items, H, nT, stride, scale_log2
  const float* q_scale;         // [B*H] dequantisation scales
  const float* k_scale;
  const float* v_scale;
};

// TMA producer of Q (per item) and K_j (kKSt-deep ring), plus a record per block.
__device__ __forceinline__ void role_qk_producer(const attn::Args& a, Bars& bars, uint32_t sb,
                                                 const CUtensorMap* tmQ, const CUtensorMap* tmK,
                                                 volatile int* abort) {
  uint32_t kc = 0, qc = 0;
  bool stop = false;
  for (int64_t mm = 0; !stop; ++mm) {
    const int64_t u = cta_item(mm);
    if (u >= a.items) break;
    int32_t nf;
    bool bad;
    const int32_t n = item_blocks(a, u, nf, bad);
    if (n == 0) continue;
    const uint32_t qb = qc % kQSt;
    if (qc >= kQSt && !mbar_wait(smem_u32(&bars.q_empty[qb]), (qc / kQSt - 1) & 1, abort, 110)) break;
    const uint32_t qbar = smem_u32(&bars.q_full[qb]);
    mbar_arrive_expect_tx(qbar, kTileB);
    tma_load_2d(sb + kOffQ + qb * kTileB, tmQ, qbar, 0, static_cast<int32_t>(u * 128));
    const int64_t head_row = (u / a.nT) * a.nT;
    const int32_t* valid_h = a.valid + ((u / a.nT) % a.H) * a.nT;
    const int32_t d = diag_pos(a, u, nf, n);
    for (int32_t j = 0; j < n; ++j) {
      bool b2;
      const int32_t jj = visit_pos(j, d);
      const int32_t idx = item_key(a, u, nf, jj, b2);
      if (b2) flag_status(ST_BAD_LIST);
      const int32_t row = static_cast<int32_t>((head_row + idx) * 128);
      const uint32_t ks = kc % kKSt;
      if (kc >= kKSt && !mbar_wait(smem_u32(&bars.k_empty[ks]), (kc / kKSt - 1) & 1, abort, 111)) { stop = true; break; }
      bars.k_op[ks] = (j == 0 ? kOpNewItem : 0u) | (j == n - 1 ? kOpLastBlk : 0u) | (qb << kOpQBufShift);
      const uint32_t kb = smem_u32(&bars.k_full[ks]);
      mbar_arrive_expect_tx(kb, kTileB);
      tma_load_2d(sb + kOffK + ks * kTileB, tmK, kb, 0, row);
      int32_t nv = 128;
      if (jj >= nf) {
        nv = valid_h[idx];
        if (nv < 1 || nv > 128) {
          flag_status(ST_BAD_LIST);
          nv = nv < 1 ? 1 : 128;
        }
      }
      bars.rec_nv[kc % kRec] = nv;
      bars.rec_idx[kc % kRec] = idx;
      mbar_arrive(smem_u32(&bars.rec_full[kc % kRec]));
      ++kc;
    }
    ++qc;
  }
  if (!*abort) {
    const uint32_t ks = kc % kKSt;
    if (kc < kKSt || mbar_wait(smem_u32(&bars.k_empty[ks]), (kc / kKSt - 1) & 1, abort, 112)) {
      bars.k_op[ks] = kOpStop;
      mbar_arrive(smem_u32(&bars.k_full[ks]));
    }
  }
  if (*abort) {
    for (uint32_t i = kc > kKSt ? kc - kKSt : 0; i < kc; ++i)
      mbar_wait(smem_u32(&bars.k_full[i % kKSt]), (i / kKSt) & 1, nullptr, 113);
    for (uint32_t i = qc > kQSt ? qc - kQSt : 0; i < qc; ++i)
      mbar_wait(smem_u32(&bars.q_full[i % kQSt]), (i / kQSt) & 1, nullptr, 114);
  }
}

// TMA producer of the transposed V tiles (kVSt-deep ring).
__device__ __forceinline__ void role_v_producer(const attn::Args& a, Bars& bars, uint32_t sb, const CUtensorMap* tmV,
                                                volatile int* abort) {
  uint32_t vc = 0, items = 0;
  bool stop = false;
  for (int64_t mm = 0; !stop; ++mm) {
    const int64_t u = cta_item(mm);
    if (u >= a.items) break;
    int32_t nf;
    bool bad;
    const int32_t n = item_blocks(a, u, nf, bad);
    if (n == 0) continue;
    const int64_t head_row = (u / a.nT) * a.nT;
    const int32_t d = diag_pos(a, u, nf, n);
    for (int32_t j = 0; j < n; ++j) {
      bool b2;
      const int32_t idx = item_key(a, u, nf, visit_pos(j, d), b2);
      const int32_t row = static_cast<int32_t>((head_row + idx) * 128);
      const uint32_t vs = vc % kVSt;
      if (vc >= kVSt && !mbar_wait(smem_u32(&bars.v_empty[vs]), (vc / kVSt - 1) & 1, abort, 115)) { stop = true; break; }
      bars.v_op[vs] = (j == 0 ? kOpNewItem : 0u) | (j == n - 1 ? kOpLastBlk : 0u) | (items == 0 ? kOpFirstItem : 0u);
      const uint32_t vb = smem_u32(&bars.v_full[vs]);
      mbar_arrive_expect_tx(vb, kTileB);
      tma_load_2d(sb + kOffV + vs * kTileB, tmV, vb, 0, row);
      ++vc;
    }
    ++items;
  }
  if (!*abort) {
    const uint32_t vs = vc % kVSt;
    if (vc < kVSt || mbar_wait(smem_u32(&bars.v_empty[vs]), (vc / kVSt - 1) & 1, abort, 116)) {
      bars.v_op[vs] = kOpStop;
      mbar_arrive(smem_u32(&bars.v_full[vs]));
    }
  }
  if (*abort) {
    for (uint32_t i = vc > kVSt ? vc - kVSt : 0; i < vc; ++i)
      mbar_wait(smem_u32(&bars.v_full[i % kVSt]), (i / kVSt) & 1, nullptr, 117);
  }
}

// Q K^T issuer: S_b = Q K_j^T (four K32 e4m3 MMAs) once every softmax warp has taken S(j-2).
__device__ __forceinline__ void role_qk_issuer(Bars& bars, uint32_t sb, uint32_t tmem, volatile int* abort) {
  // one 128-byte row per tile row holds all 128 channels: a k-step of 32 channels moves the
  // start address by 32 bytes (2 in the 16-byte field) inside the swizzle atom
  const uint64_t dQ = smem_desc_sw128(sb + kOffQ, 16, 1024);
  const uint64_t dK = smem_desc_sw128(sb + kOffK, 16, 1024);
  uint32_t qn[kQSt];
  for (int i = 0; i < kQSt; ++i) qn[i] = 0;
  for (uint32_t g = 0;; ++g) {
    const uint32_t ks = g % kKSt;
    if (!mbar_wait(smem_u32(&bars.k_full[ks]), (g / kKSt) & 1, abort, 118)) break;
    const uint32_t op = bars.k_op[ks];
    if (op & kOpStop) break;
    const uint32_t qb = op >> kOpQBufShift;
    if (op & kOpNewItem) {
      if (!mbar_wait(smem_u32(&bars.q_full[qb]), qn[qb] & 1, abort, 119)) break;
      ++qn[qb];
    }
    const uint32_t sbuf = g & 1;
    if (g >= 2 && !mbar_wait(smem_u32(&bars.s_free[sbuf]), ((g >> 1) - 1) & 1, abort, 120)) break;
    tc_fence_after();
    const uint64_t a0 = opaque(dQ + static_cast<uint64_t>(qb * (kTileB >> 4)));
    const uint64_t b0 = opaque(dK + static_cast<uint64_t>(ks * (kTileB >> 4)));
    const uint32_t d = tmem + kColS + sbuf * 128;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_ss_f8(d, a0 + static_cast<uint64_t>(kk * 2), b0 + static_cast<uint64_t>(kk * 2), kIdesc, kk > 0 ? 1u : 0u);
    tc_commit(smem_u32(&bars.s_full[sbuf]));
    if (op & kOpLastBlk) tc_commit(smem_u32(&bars.q_empty[qb]));
    tc_commit(smem_u32(&bars.k_empty[ks]));
  }
  tc_commit(smem_u32(&bars.drain[0]));
  mbar_wait(smem_u32(&bars.drain[0]), 0, nullptr, 121);
}

// P V issuer: O += P_b (tensor memory, e4m3, 8 columns per K = 32 step) x V_j (transposed
// tile, K-major).
__device__ __forceinline__ void role_pv_issuer(Bars& bars, uint32_t sb, uint32_t tmem, volatile int* abort) {
  const uint64_t dV = smem_desc_sw128(sb + kOffV, 16, 1024);
  uint32_t items_done = 0;
  for (uint32_t g = 0;; ++g) {
    const uint32_t vs = g % kVSt;
    if (!mbar_wait(smem_u32(&bars.v_full[vs]), (g / kVSt) & 1, abort, 122)) break;
    const uint32_t op = bars.v_op[vs];
    if (op & kOpStop) break;
    const uint32_t pb = g & 1;
    if (!mbar_wait(smem_u32(&bars.p_full[pb]), (g >> 1) & 1, abort, 123)) break;
    if ((op & kOpNewItem) && !(op & kOpFirstItem) &&
        !mbar_wait(smem_u32(&bars.o_free), (items_done - 1) & 1, abort, 124))
      break;
    tc_fence_after();
    const uint32_t pa = tmem + kColP + pb * 32;
    const uint64_t b0 = opaque(dV + static_cast<uint64_t>(vs * (kTileB >> 4)));
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_ts_f8(tmem + kColO, pa + kk * 8, b0 + static_cast<uint64_t>(kk * 2), kIdesc,
                (kk > 0 || !(op & kOpNewItem)) ? 1u : 0u);
    tc_commit(smem_u32(&bars.o_done[pb]));
    tc_commit(smem_u32(&bars.v_empty[vs]));
    if (op & kOpLastBlk) ++items_done;
  }
  tc_commit(smem_u32(&bars.drain[1]));
  mbar_wait(smem_u32(&bars.drain[1]), 0, nullptr, 125);
}

// Column groups k (bit k) whose exponentials run on the FMA pipe (exp2_fma_x2) instead of
// the MUFU, for a thread's first row (r0) and second row (r0 + 8): the MUFU sets the pace of
// this softmax while the FMA pipe is mostly idle. An eighth of the exponentials (measured at
// the 16:9 clip: none 7.85 ms, 1/8 7.52, 1/4 7.60, 3/8 8.27, 1/2 8.82).
constexpr uint32_t kFmaExpRow0 = 0x0000u;
constexpr uint32_t kFmaExpRow1 = 0x8888u;

// Softmax warps: the bf16 kernel's 16-row layout (thread: rows r0 = base + lane / 4 and
// r0 + 8, of every 8-column group k the columns 8k + 2c + {0, 1}, c = lane % 4). One pass
// takes the exponentials with the block's row maxima; P goes to tensor memory as e4m3 words.
__device__ __forceinline__ void softmax_role(const Args& p, Bars& bars, uint32_t tmem, uint32_t warp,
                                             uint32_t lane) {
  using namespace attn;
  const attn::Args& a = p.a;
  volatile int* abort = &bars.abort;
  const uint32_t base = 32 * (warp & 3) + 16 * (warp >> 2);
  const uint32_t lane_off = base << 16;
  const uint32_t r0 = base + lane / 4, c = lane & 3;
  uint32_t g = 0;
  for (int64_t mm = 0;; ++mm) {
    const int64_t u = cta_item(mm);
    if (u >= a.items) break;
    int32_t nf;
    bool bad;
    const int32_t n = item_blocks(a, u, nf, bad);
    __nv_bfloat16* orow0 = a.o + (u * 128 + r0) * 128;
    __nv_bfloat16* orow1 = orow0 + 8 * 128;
    if (n == 0) {
      if (bad && lane == 0 && warp == 0) flag_status(ST_BAD_LIST);
      uint4* z0 = reinterpret_cast<uint4*>(orow0 + c * 32);
      uint4* z1 = reinterpret_cast<uint4*>(orow1 + c * 32);
#pragma unroll
      for (int i = 0; i < 4; ++i) { z0[i] = make_uint4(0, 0, 0, 0); z1[i] = make_uint4(0, 0, 0, 0); }
      if (a.lse && c == 0) { a.lse[u * 128 + r0] = -INFINITY; a.lse[u * 128 + r0 + 8] = -INFINITY; }
      continue;
    }
    const int64_t bh = u / a.nT;
    const float cs = a.scale_log2 * p.q_scale[bh] * p.k_scale[bh];   // score -> log2 units
    const uint64_t c2 = f2_pack(__float_as_uint(cs), __float_as_uint(cs));
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    bool ok = true;
    for (int32_t j = 0; j < n; ++j, ++g) {
      const uint32_t sbuf = g & 1;
      if (!warp_wait_abort(smem_u32(&bars.rec_full[g % kRec]), (g / kRec) & 1, abort, 126)) { ok = false; break; }
      const int32_t nv = reinterpret_cast<volatile int32_t*>(bars.rec_nv)[g % kRec];
      if (!warp_wait_abort(smem_u32(&bars.s_full[sbuf]), (g >> 1) & 1, abort, 127)) { ok = false; break; }
      tc_fence_after();
      uint32_t s[64];
      tmem_ld_16x256b_x16(tmem + lane_off + kColS + sbuf * 128, s);
      tmem_wait_ld();
      reg_fence(s);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars.s_free[sbuf]));
      if (nv < 128) {
        const int32_t kv0 = (nv - 2 * static_cast<int32_t>(c) + 7) >> 3;
        const int32_t kv1 = (nv - 2 * static_cast<int32_t>(c) + 6) >> 3;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          if (k >= kv0) { s[4 * k] = 0xFF800000u; s[4 * k + 2] = 0xFF800000u; }
          if (k >= kv1) { s[4 * k + 1] = 0xFF800000u; s[4 * k + 3] = 0xFF800000u; }
        }
      }
      // Exponentials with the current reference m, computed together with the block's row
      // maxima (one basic block, so the MUFU and max chains interleave). If a row's maximum
      // (log2 units) grew by more than 1.75, 2^7 P may have passed e4m3's range: the reference
      // moves, O is rescaled and the pass is repeated. The roles visit the diagonal key tile
      // first, which holds most rows' maxima, so repeats are rare. Block 0 of an item takes
      // its row maxima first, so that its single pass has a reference.
      if (j == 0) {
        float a4[4], b4[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          a4[q] = fmaxf(__uint_as_float(s[4 * q]), __uint_as_float(s[4 * q + 1]));
          b4[q] = fmaxf(__uint_as_float(s[4 * q + 2]), __uint_as_float(s[4 * q + 3]));
        }
#pragma unroll
        for (int k = 4; k < 16; ++k) {
          a4[k & 3] = fmax3(a4[k & 3], __uint_as_float(s[4 * k]), __uint_as_float(s[4 * k + 1]));
          b4[k & 3] = fmax3(b4[k & 3], __uint_as_float(s[4 * k + 2]), __uint_as_float(s[4 * k + 3]));
        }
        m0 = quad_max(fmaxf(fmaxf(a4[0], a4[1]), fmaxf(a4[2], a4[3]))) * cs;
        m1 = quad_max(fmaxf(fmaxf(b4[0], b4[1]), fmaxf(b4[2], b4[3]))) * cs;
      }
      // 2^(s * cs - m + 7) -> e4m3. Word m of a row (column 4m + c of the P buffer, 16x128b
      // shape) packs the pairs of 8-column groups 2m and 2m + 1: key slots 16m + 2c + {0, 1}
      // and 16m + 8 + 2c + {0, 1}, the order of V's transposed tiles
      uint32_t pk[16];
      uint64_t acc0[2], acc1[2];
#pragma unroll 1
      for (int pass = 0;; ++pass) {
        const uint64_t nm0 = f2_pack(__float_as_uint(kPExp - m0), __float_as_uint(kPExp - m0));
        const uint64_t nm1 = f2_pack(__float_as_uint(kPExp - m1), __float_as_uint(kPExp - m1));
        acc0[0] = acc0[1] = acc1[0] = acc1[1] = 0ull;
        float a4[4], b4[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          a4[q] = fmaxf(__uint_as_float(s[4 * q]), __uint_as_float(s[4 * q + 1]));
          b4[q] = fmaxf(__uint_as_float(s[4 * q + 2]), __uint_as_float(s[4 * q + 3]));
        }
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          if (k >= 4) {
            a4[k & 3] = fmax3(a4[k & 3], __uint_as_float(s[4 * k]), __uint_as_float(s[4 * k + 1]));
            b4[k & 3] = fmax3(b4[k & 3], __uint_as_float(s[4 * k + 2]), __uint_as_float(s[4 * k + 3]));
          }
          const uint64_t xx = f2_fma(f2_pack(s[4 * k], s[4 * k + 1]), c2, nm0);
          const uint64_t yy = f2_fma(f2_pack(s[4 * k + 2], s[4 * k + 3]), c2, nm1);
          float p0, p1, q0, q1;
          if ((kFmaExpRow0 >> k) & 1) {
            exp2_fma_x2(xx, p0, p1);
          } else {
            f2_unpack(xx, p0, p1);
            p0 = ex2_approx(p0);
            p1 = ex2_approx(p1);
          }
          if ((kFmaExpRow1 >> k) & 1) {
            exp2_fma_x2(yy, q0, q1);
          } else {
            f2_unpack(yy, q0, q1);
            q0 = ex2_approx(q0);
            q1 = ex2_approx(q1);
          }
          acc0[k & 1] = f2_add(acc0[k & 1], f2_pack(__float_as_uint(p0), __float_as_uint(p1)));
          acc1[k & 1] = f2_add(acc1[k & 1], f2_pack(__float_as_uint(q0), __float_as_uint(q1)));
          const uint32_t e0 = pack_e4m3x2(p0, p1), e1 = pack_e4m3x2(q0, q1);
          if (k & 1) {
            pk[k - 1] |= e0 << 16;
            pk[k] |= e1 << 16;
          } else {
            pk[k] = e0;
            pk[k + 1] = e1;
          }
        }
        const float mb0 = quad_max(fmaxf(fmaxf(a4[0], a4[1]), fmaxf(a4[2], a4[3]))) * cs;
        const float mb1 = quad_max(fmaxf(fmaxf(b4[0], b4[1]), fmaxf(b4[2], b4[3]))) * cs;
        const bool need0 = mb0 > m0 + kRescaleLog2, need1 = mb1 > m1 + kRescaleLog2;
        if (pass == 1 || !__any_sync(0xffffffffu, need0 || need1)) break;
        // O must hold P V of every earlier block before it is rescaled
        const uint32_t gp = g - 1;
        if (!warp_wait_abort(smem_u32(&bars.o_done[gp & 1]), (gp >> 1) & 1, abort, 128)) { ok = false; break; }
        tc_fence_after();
        const float al0 = need0 ? ex2_approx(m0 - mb0) : 1.0f;
        const float al1 = need1 ? ex2_approx(m1 - mb1) : 1.0f;
        const uint64_t al0x2 = f2_pack(__float_as_uint(al0), __float_as_uint(al0));
        const uint64_t al1x2 = f2_pack(__float_as_uint(al1), __float_as_uint(al1));
#pragma unroll 1
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t o16[16];
          const uint32_t oa = tmem + lane_off + kColO + ch * 32;
          tmem_ld_16x256b_x4(oa, o16);
          tmem_wait_ld();
          reg_fence(o16);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float x, y;
            f2_unpack(f2_mul(f2_pack(o16[4 * q], o16[4 * q + 1]), al0x2), x, y);
            o16[4 * q] = __float_as_uint(x); o16[4 * q + 1] = __float_as_uint(y);
            f2_unpack(f2_mul(f2_pack(o16[4 * q + 2], o16[4 * q + 3]), al1x2), x, y);
            o16[4 * q + 2] = __float_as_uint(x); o16[4 * q + 3] = __float_as_uint(y);
          }
          tmem_st_16x256b_x4(oa, o16);
        }
        tmem_wait_st();
        if (need0) { l0 *= al0; m0 = mb0; }
        if (need1) { l1 *= al1; m1 = mb1; }
      }
      if (!ok) break;
      {
        float t0, t1, t2, t3;
        f2_unpack(acc0[0], t0, t1); f2_unpack(acc0[1], t2, t3);
        l0 += (t0 + t1) + (t2 + t3);
        f2_unpack(acc1[0], t0, t1); f2_unpack(acc1[1], t2, t3);
        l1 += (t0 + t1) + (t2 + t3);
      }
      // P buffer g & 1 is free once P V of block g - 2 has completed
      if (g >= 2) {
        const uint32_t gp = g - 2;
        if (!warp_wait_abort(smem_u32(&bars.o_done[gp & 1]), (gp >> 1) & 1, abort, 129)) { ok = false; break; }
        tc_fence_after();
      }
      tmem_st_16x128b_x8(tmem + lane_off + kColP + sbuf * 32, pk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars.p_full[sbuf]));
    }
    if (!ok) break;
    // epilogue: O * v_scale / l -> bf16, LSE
    const float lt0 = quad_sum(l0), lt1 = quad_sum(l1);
    const uint32_t gl = g - 1;
    if (!warp_wait_abort(smem_u32(&bars.o_done[gl & 1]), (gl >> 1) & 1, abort, 130)) break;
    tc_fence_after();
    const float sv = p.v_scale[bh];
    const float inv0 = sv / lt0, inv1 = sv / lt1;
#pragma unroll
    for (int ch = 0; ch < 4; ++ch) {
      uint32_t o16[16];
      tmem_ld_16x256b_x4(tmem + lane_off + kColO + ch * 32, o16);
      tmem_wait_ld();
      reg_fence(o16);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int col = ch * 32 + 8 * q + 2 * static_cast<int>(c);
        *reinterpret_cast<uint32_t*>(orow0 + col) =
            pack_bf16x2(__uint_as_float(o16[4 * q]) * inv0, __uint_as_float(o16[4 * q + 1]) * inv0);
        *reinterpret_cast<uint32_t*>(orow1 + col) =
            pack_bf16x2(__uint_as_float(o16[4 * q + 2]) * inv1, __uint_as_float(o16[4 * q + 3]) * inv1);
      }
    }
    if (a.lse && c == 0) {
      a.lse[u * 128 + r0] = (m0 - kPExp + __log2f(lt0)) * kLn2;
      a.lse[u * 128 + r0 + 8] = (m1 - kPExp + __log2f(lt1)) * kLn2;
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&bars.o_free));
  }
}

__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_fp8_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const Args p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ Bars bars;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const uint32_t tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, wg = warp >> 2;
  volatile int* abort = &bars.abort;

  if (tid == 0) attn::init_bars(bars);
  if (warp == 9) {
    tmem_alloc(smem_u32(&bars.tmem_base), kTmemCols);
    tmem_relinquish();
  }
  if ((warp == 8 || warp == 11) && lane == 0) {
    prefetch_tensormap(&tmQ);
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;

  if (wg == 2) {
    attn::reg_dealloc<attn::kControlRegs>();
    if (warp == 8 && lane == 0)
      fp8::role_qk_producer(p.a, bars, sb, &tmQ, &tmK, abort);
    else if (warp == 11 && lane == 0)
      fp8::role_v_producer(p.a, bars, sb, &tmV, abort);
    else if (warp == 9 && lane == 0)
      fp8::role_qk_issuer(bars, sb, tmem, abort);
    else if (warp == 10 && lane == 0)
      fp8::role_pv_issuer(bars, sb, tmem, abort);
  } else {
    attn::reg_alloc<attn::kSoftmaxRegs>();
    fp8::softmax_role(p, bars, tmem, warp, lane);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace fp8
}  // namespace veda
