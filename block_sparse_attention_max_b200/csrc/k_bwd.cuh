// k_bwd.cuh -- backward of the block-sparse attention forward over the same block lists.
//
// "Miowtion" README, Key Features / Veda sparse attention: the block-sparse integration
// carries "transposed backward lists". For an output gradient dO, per query row q over the
// forward's keys: P = exp(scale q.k - LSE_q), D_q = dO_q . O_q, dS = P (dO_q . v - D_q),
// dQ_q = scale sum_k dS k, dK_k += scale sum_q dS q, dV_k += sum_q P dO_q.
//
// Three launches:
//   delta_kernel           D = rowsum(dO * O) per query row (HBM stream)
//   transpose_lists_kernel query tiles of every key tile (one warp per key tile)
//   bwd_kernel<kModeDQ>    one query tile per CTA item, over its forward list: S = Q K_j^T,
//                          dP = dO V_j^T, dS in TMEM, dQ += dS K_j (a key tile with at most
//                          64 valid slots over its first 64 keys only, as in the forward)
//   bwd_kernel<kModeDKDV>  one key tile per CTA item, over its transposed list:
//                          S^T = K Q_i^T, dP^T = V dO_i^T, P^T and dS^T in TMEM,
//                          dV += P^T dO_i, dK += dS^T Q_i
// Both modes share the structure: per item two "fixed" tiles (Q, dO or K, V), per block two
// "streamed" tiles (K_j, V_j or Q_i, dO_i) in a 2-slot ring; the two score-like MMAs are
// fixed x streamed^T (shared-memory operands, K-major); the accumulating MMAs read their A
// operand (dS, P^T, dS^T as bf16) from tensor memory and the streamed tile as an MN-major B
// operand. Tensor memory: S | dP | acc0 | acc1 (128 columns each). The eight softmax warps
// use the forward's 16-lane layout (16 rows per warp, rows r0 and r0 + 8 per thread).
// The MMAs of the next block of an item are issued ahead of the current block's
// accumulating MMAs wherever tensor memory allows, so the tensor core works while the
// softmax does (one issuing thread: its MMAs run in issue order, so an MMA that overwrites
// S or dP always follows the MMA that reads what the softmax wrote there):
//   dQ:    S has two buffers (the fourth 128-column block is free in this mode); per block
//          ... dP(j+1) [once the softmax has read dP(j)], dQ(j) [dS(j) written], S(j+2) ...
//   dK/dV: the softmax hands over in two steps, P^T (exponentials only) and then dS^T
//          (once dP^T has landed); per block ... dV(j) [P^T(j)], S^T(j+1), dK(j) [dS^T(j)],
//          dP^T(j+1) ... so the exponentials of block j+1 overlap dK(j) and dP^T(j+1).
#pragma once

#include "k_attn.cuh"

namespace veda {
namespace bwd {

using attn::kThreads;
using attn::kTileB;
using attn::kHalfB;

constexpr int kModeDQ = 0;
constexpr int kModeDKDV = 1;
// Streamed tiles in two rings: ring A holds the tile whose last reader is the block's late
// accumulating MMA (dQ: K_j, read by dQ(j); dK/dV: Q_i, read by dK(j)), ring B the one whose
// last reader comes early (dQ: V_j, read by dP(j); dK/dV: dO_i, read by dV(j)), so ring A
// gets the extra slot: a slot is refilled only after its last reader, and a 32 KB tile
// takes ~1,400 cycles to arrive from L2.
constexpr int kStA = 3;                         // ring A slots
constexpr int kStB = 2;                         // ring B slots
constexpr int kStStat = 2;                      // dK/dV: LSE + D rows of the streamed query tiles
constexpr uint32_t kStatB = 1024;
constexpr uint32_t kOffFix = 0;                 // two fixed tiles
constexpr uint32_t kOffA = 2 * kTileB;
constexpr uint32_t kOffB = kOffA + kStA * kTileB;
constexpr uint32_t kOffStat = kOffB + kStB * kTileB;            // 224 KB
// dQ: the tiles plus 1 KB of alignment slack; dK/dV: the tiles and the stats ring exactly
// (226 KB, which with the static barriers is the 227 KB a block may have), so that kernel
// checks that its dynamic shared memory starts 1024-byte aligned and does no work otherwise
constexpr uint32_t kSmemBytesDQ = kOffStat + 1024;
constexpr uint32_t kSmemBytesDKDV = kOffStat + kStStat * kStatB;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColDP = 128, kColA0 = 256, kColA1 = 384;
constexpr uint32_t kColS1 = 384;                // dQ mode: second S buffer (acc1 unused)
constexpr uint32_t kIdescSS = idesc_bf16_f32(128, 128, 0, 0);   // A, B K-major
constexpr uint32_t kIdescSS64 = idesc_bf16_f32(128, 64, 0, 0);  // the first 64 keys (dQ mode)
constexpr uint32_t kIdescTS = idesc_bf16_f32(128, 128, 0, 1);   // B MN-major
constexpr int kRec = 8;
constexpr int kItemRec = 4;                     // item records (dynamic work queue)
constexpr float kLog2e = 1.4426950408889634f;

struct Args {
  const int32_t* valid;         // [H][nT]
  // lists of the item: the forward's (dQ: full + partial) or the transposed ones (dK/dV:
  // full only, part_cnt == nullptr)
  const int32_t* full_cnt;
  const int32_t* full_idx;
  const int32_t* part_cnt;
  const int32_t* part_idx;
  int32_t stride;
  const float* lse;             // [B*H*nT*128] natural-log LSE of the forward
  const float* delta;           // [B*H*nT*128] D = rowsum(dO * O)
  __nv_bfloat16* out0;          // dQ (dQ mode) or dV (dK/dV mode) [B*H*nT*128][128]
  __nv_bfloat16* out1;          // dK (dK/dV mode)
  int32_t H, nT;
  int64_t items;                // B*H*nT
  float scale;                  // softmax scale
  int32_t* next_item;           // work-queue counter, zeroed before the launch
};

struct Bars {
  uint64_t fix_full, fix_empty;
  uint64_t a_full[kStA], a_empty[kStA], b_full[kStB], b_empty[kStB];
  uint64_t st_full[kStStat], st_empty[kStStat];
  uint64_t s_full[2];            // S-like MMA of block g landed (dQ: buffer g & 1; dK/dV: [0])
  uint64_t dp_full, dp_free;     // dP-like MMA landed / the softmax holds dP (dQ) in registers
  uint64_t pa_full;              // softmax wrote P^T over S^T (dK/dV)
  // softmax wrote dS over S (dQ: one barrier per S buffer, since the softmax may finish
  // block g + 1 before the issuer has looked at block g) or dS^T over dP^T (dK/dV: [0])
  uint64_t pb_full[2];
  uint64_t o_done, o_free, drain;
  uint64_t rec_full[kRec];
  int32_t rec_nv[kRec];
  // items are taken from a global counter by the producer (transposed lists are very
  // uneven: a popular key tile is listed by hundreds of query tiles) and handed to the
  // softmax warps through these records (-1 = no more work)
  uint64_t item_full[kItemRec], item_free[kItemRec];
  int32_t item_u[kItemRec];
  uint32_t a_op[kStA];                 // block flags, written with the ring-A tile
  uint32_t tmem_base;
  int32_t abort;
};

// kOpHalf (dQ mode): the streamed key tile has at most 64 valid slots; S, dP and dQ's
// accumulation run over its first 64 keys only (pad key slots get no gradient anyway).
enum : uint32_t { kOpNewItem = 1u, kOpLastBlk = 2u, kOpFirstItem = 4u, kOpStop = 8u, kOpHalf = 16u };

__device__ __forceinline__ int32_t list_len(const Args& a, int64_t u, int32_t& nf, bool& bad) {
  nf = a.full_cnt[u];
  const int32_t np = a.part_cnt ? a.part_cnt[u] : 0;
  bad = nf < 0 || np < 0 || nf > a.stride || np > a.stride || nf + np > a.nT;
  if (bad) { nf = 0; return 0; }
  return nf + np;
}
__device__ __forceinline__ int32_t list_at(const Args& a, int64_t u, int32_t nf, int32_t j, bool& bad) {
  const int32_t idx = j < nf ? a.full_idx[u * a.stride + j] : a.part_idx[u * a.stride + (j - nf)];
  bad = idx < 0 || idx >= a.nT;
  return bad ? 0 : idx;
}

// ---------------------------------------------------------------- producer (one thread)
template <int MODE>
__device__ __forceinline__ void role_producer(const Args& a, Bars& bars, uint32_t sb, const CUtensorMap* tmF0,
                                              const CUtensorMap* tmF1, const CUtensorMap* tmS0,
                                              const CUtensorMap* tmS1, volatile int* abort) {
  uint32_t sc = 0, fc = 0;
  uint32_t na = 0, nb = 0, ns = 0;   // copies issued into ring A, ring B and the stats ring
  bool stop = false;
  for (uint32_t ic = 0; !stop; ++ic) {
    const uint32_t is = ic % kItemRec;
    if (ic >= kItemRec && !mbar_wait(smem_u32(&bars.item_free[is]), (ic / kItemRec - 1) & 1, abort, 54)) break;
    const int64_t u = atomicAdd(a.next_item, 1);
    bars.item_u[is] = u < a.items ? static_cast<int32_t>(u) : -1;
    mbar_arrive(smem_u32(&bars.item_full[is]));
    if (u >= a.items) break;
    int32_t nf;
    bool bad;
    const int32_t n = list_len(a, u, nf, bad);
    if (n == 0) continue;
    if (fc > 0 && !mbar_wait(smem_u32(&bars.fix_empty), (fc - 1) & 1, abort, 40)) break;
    const uint32_t fb = smem_u32(&bars.fix_full);
    mbar_arrive_expect_tx(fb, 2 * kTileB);
    const int32_t frow = static_cast<int32_t>(u * 128);
    tma_load_2d(sb + kOffFix, tmF0, fb, 0, frow);
    tma_load_2d(sb + kOffFix + kHalfB, tmF0, fb, 64, frow);
    tma_load_2d(sb + kOffFix + kTileB, tmF1, fb, 0, frow);
    tma_load_2d(sb + kOffFix + kTileB + kHalfB, tmF1, fb, 64, frow);
    const int64_t head_row = (u / a.nT) * a.nT;
    const int32_t* valid_h = a.valid + ((u / a.nT) % a.H) * a.nT;
    for (int32_t j = 0; j < n; ++j) {
      bool b2;
      const int32_t idx = list_at(a, u, nf, j, b2);
      if (b2) flag_status(ST_BAD_LIST);
      const int64_t t = head_row + idx;                 // streamed tile (b, h, idx)
      const int32_t srow = static_cast<int32_t>(t * 128);
      // ring A: tile 0 of the block, plus its flags
      const uint32_t sa = sc % kStA;
      if (sc >= kStA && !mbar_wait(smem_u32(&bars.a_empty[sa]), (sc / kStA - 1) & 1, abort, 41)) {
        stop = true;
        break;
      }
      // dQ mode: valid key slots of the streamed key tile (the softmax's record, the half flag)
      int32_t nv = 128;
      if (MODE == kModeDQ) {
        nv = valid_h[idx];
        if (nv < 0 || nv > 128) {
          flag_status(ST_BAD_LIST);
          nv = nv < 0 ? 0 : 128;
        }
      }
      bars.a_op[sa] = (j == 0 ? kOpNewItem : 0u) | (j == n - 1 ? kOpLastBlk : 0u) | (fc == 0 ? kOpFirstItem : 0u) |
                      (MODE == kModeDQ && nv <= 64 ? kOpHalf : 0u);
      {
        const uint32_t dst = sb + kOffA + sa * kTileB;
        const uint32_t bar = smem_u32(&bars.a_full[sa]);
        mbar_arrive_expect_tx(bar, kTileB);
        tma_load_2d(dst, tmS0, bar, 0, srow);
        tma_load_2d(dst + kHalfB, tmS0, bar, 64, srow);
        ++na;
      }
      // ring B: tile 1 of the block
      const uint32_t sbb = sc % kStB;
      if (sc >= kStB && !mbar_wait(smem_u32(&bars.b_empty[sbb]), (sc / kStB - 1) & 1, abort, 64)) {
        stop = true;
        break;
      }
      {
        const uint32_t dst = sb + kOffB + sbb * kTileB;
        const uint32_t bar = smem_u32(&bars.b_full[sbb]);
        mbar_arrive_expect_tx(bar, kTileB);
        tma_load_2d(dst, tmS1, bar, 0, srow);
        tma_load_2d(dst + kHalfB, tmS1, bar, 64, srow);
        ++nb;
      }
      if (MODE == kModeDKDV) {
        // the streamed query tile's LSE and D rows (512 B each, 16-byte aligned)
        const uint32_t st = sc % kStStat;
        if (sc >= kStStat && !mbar_wait(smem_u32(&bars.st_empty[st]), (sc / kStStat - 1) & 1, abort, 65)) {
          stop = true;
          break;
        }
        const uint32_t dst = sb + kOffStat + st * kStatB;
        const uint32_t bar = smem_u32(&bars.st_full[st]);
        mbar_arrive_expect_tx(bar, kStatB);
        bulk_g2s(dst, a.lse + t * 128, 512, bar);
        bulk_g2s(dst + 512, a.delta + t * 128, 512, bar);
        ++ns;
      }
      if (MODE == kModeDQ) {
        // block record for the softmax: valid key slots of the streamed key tile (entry
        // sc % kRec was last read for block sc - kRec, long before ring-A slot sc - kStA came back)
        bars.rec_nv[sc % kRec] = nv;
        mbar_arrive(smem_u32(&bars.rec_full[sc % kRec]));
      }
      ++sc;
    }
    ++fc;
  }
  if (!*abort) {
    const uint32_t sa = sc % kStA;
    if (sc < kStA || mbar_wait(smem_u32(&bars.a_empty[sa]), (sc / kStA - 1) & 1, abort, 42)) {
      bars.a_op[sa] = kOpStop;
      mbar_arrive(smem_u32(&bars.a_full[sa]));
    }
  }
  if (*abort) {
    // let the copies this thread issued land before the CTA exits, ring by ring
    for (uint32_t i = na > kStA ? na - kStA : 0; i < na; ++i)
      mbar_wait(smem_u32(&bars.a_full[i % kStA]), (i / kStA) & 1, nullptr, 43);
    for (uint32_t i = nb > kStB ? nb - kStB : 0; i < nb; ++i)
      mbar_wait(smem_u32(&bars.b_full[i % kStB]), (i / kStB) & 1, nullptr, 66);
    for (uint32_t i = ns > kStStat ? ns - kStStat : 0; i < ns; ++i)
      mbar_wait(smem_u32(&bars.st_full[i % kStStat]), (i / kStStat) & 1, nullptr, 67);
    if (fc > 0) mbar_wait(smem_u32(&bars.fix_full), (fc - 1) & 1, nullptr, 44);
  }
}

// ---------------------------------------------------------------- MMA issuer (one thread)
// 128 x 128 x 128 products as 8 K16 MMAs: score-like F x S^T (both K-major in shared memory)
// and accumulating A (bf16 in TMEM) x S (MN-major in shared memory).
// half: the streamed tile's first 64 rows only (N = 64 for the score-like product, K = 64
// for the accumulating one).
__device__ __forceinline__ void mma_score(uint32_t d, uint64_t a0, uint64_t b0, bool half = false) {
  const uint32_t idesc = half ? kIdescSS64 : kIdescSS;
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint64_t koff = static_cast<uint64_t>((kk >> 2) * (kHalfB >> 4) + (kk & 3) * 2);
    mma_ss(d, a0 + koff, b0 + koff, idesc, kk > 0 ? 1u : 0u);
  }
}
__device__ __forceinline__ void mma_accum(uint32_t d, uint32_t a_tmem, uint64_t b0, uint32_t acc_first,
                                          bool half = false) {
  mma_ts(d, a_tmem, b0, kIdescTS, acc_first);
#pragma unroll
  for (int kk = 1; kk < 4; ++kk)
    mma_ts(d, a_tmem + kk * 8, b0 + static_cast<uint64_t>(kk * (2048 >> 4)), kIdescTS, 1u);
  if (!half) {
#pragma unroll
    for (int kk = 4; kk < 8; ++kk)
      mma_ts(d, a_tmem + kk * 8, b0 + static_cast<uint64_t>(kk * (2048 >> 4)), kIdescTS, 1u);
  }
}

template <int MODE>
__device__ __forceinline__ void role_issuer(Bars& bars, uint32_t sb, uint32_t tmem, volatile int* abort) {
  const uint64_t dF = smem_desc_sw128(sb + kOffFix, 16, 1024);          // fixed tiles, K-major
  const uint64_t dA = smem_desc_sw128(sb + kOffA, 16, 1024);            // ring A, K-major
  const uint64_t dAm = smem_desc_sw128(sb + kOffA, kHalfB, 1024);       // ring A, MN-major
  const uint64_t dB = smem_desc_sw128(sb + kOffB, 16, 1024);            // ring B, K-major
  const uint64_t dBm = smem_desc_sw128(sb + kOffB, kHalfB, 1024);       // ring B, MN-major
  const uint64_t fix1 = static_cast<uint64_t>(kTileB >> 4);
  auto offA = [](uint32_t g) { return static_cast<uint64_t>((g % kStA) * (kTileB >> 4)); };
  auto offB = [](uint32_t g) { return static_cast<uint64_t>((g % kStB) * (kTileB >> 4)); };
  auto s_col = [](uint32_t g) { return MODE == kModeDQ ? ((g & 1) ? kColS1 : kColS) : kColS; };
  // S-like = F0 x (ring-A tile)^T of block g into its S buffer; dP-like = F1 x (ring-B tile)^T
  // half flag of block g (its ring-A slot's op word, read after that slot's phase was seen)
  auto half_of = [&](uint32_t g) { return MODE == kModeDQ && (bars.a_op[g % kStA] & kOpHalf) != 0; };
  auto issue_s = [&](uint32_t g) {
    mma_score(tmem + s_col(g), attn::opaque(dF), attn::opaque(dA + offA(g)), half_of(g));
    tc_commit(smem_u32(&bars.s_full[MODE == kModeDQ ? (g & 1) : 0]));
  };
  auto issue_dp = [&](uint32_t g) {
    mma_score(tmem + kColDP, attn::opaque(dF + fix1), attn::opaque(dB + offB(g)), half_of(g));
    tc_commit(smem_u32(&bars.dp_full));
    if (MODE == kModeDQ) tc_commit(smem_u32(&bars.b_empty[g % kStB]));   // V_g: last reader
  };
  auto wait_a = [&](uint32_t g, uint32_t site) {
    return mbar_wait(smem_u32(&bars.a_full[g % kStA]), (g / kStA) & 1, abort, site);
  };
  auto wait_b = [&](uint32_t g, uint32_t site) {
    return mbar_wait(smem_u32(&bars.b_full[g % kStB]), (g / kStB) & 1, abort, site);
  };
  uint32_t fn = 0, items = 0;
  bool head = true;   // block g starts an item: its S / dP are not issued yet
  bool ok = true;
  for (uint32_t g = 0; ok; ++g) {
    // block g's ring-A phase was already observed before its look-ahead MMA unless it
    // starts an item (or is the stop record, which follows an item's last block)
    if (head && !wait_a(g, 45)) break;
    const uint32_t op = bars.a_op[g % kStA];
    if (op & kOpStop) break;
    if (op & kOpNewItem) {
      if (!mbar_wait(smem_u32(&bars.fix_full), fn & 1, abort, 46)) break;
      ++fn;
    }
    tc_fence_after();
    const bool last = (op & kOpLastBlk) != 0;
    if (head) {
      // dQ: dP(g) overwrites dP(g - 1), which the softmax must hold in registers by now
      if (MODE == kModeDQ && g > 0 && !mbar_wait(smem_u32(&bars.dp_free), (g - 1) & 1, abort, 60)) break;
      if (!wait_b(g, 68)) break;
      tc_fence_after();
      issue_s(g);
      issue_dp(g);
    }
    const uint32_t acc_first = (op & kOpNewItem) ? 0u : 1u;
    const bool need_o_free = (op & kOpNewItem) && !(op & kOpFirstItem);
    // the next block of the item: each of its tiles is waited for just before the MMA that
    // reads it, so that a wait overlaps MMAs already queued on the tensor core
    const uint32_t gn = g + 1;
    if (MODE == kModeDQ) {
      if (!last) {
        // S(g + 1) goes to the buffer of dS(g - 1), which dQ(g - 1), issued before, reads
        if (!wait_a(gn, 61)) break;
        tc_fence_after();
        issue_s(gn);
        // dP(g + 1) overwrites dP(g) once the softmax holds it in registers
        if (!mbar_wait(smem_u32(&bars.dp_free), g & 1, abort, 62) || !wait_b(gn, 69)) break;
        tc_fence_after();
        issue_dp(gn);
      }
      // dQ += dS (written over S(g)) x K_g (ring A, MN-major)
      if (!mbar_wait(smem_u32(&bars.pb_full[g & 1]), (g >> 1) & 1, abort, 47)) break;
      // the first accumulation of an item overwrites acc: the previous epilogue must be done
      if (need_o_free && !mbar_wait(smem_u32(&bars.o_free), (items - 1) & 1, abort, 48)) break;
      tc_fence_after();
      mma_accum(tmem + kColA0, tmem + s_col(g), attn::opaque(dAm + offA(g)), acc_first, (op & kOpHalf) != 0);
      tc_commit(smem_u32(&bars.a_empty[g % kStA]));                    // K_g: last reader
    } else {
      // dV += P^T (written over S^T) x dO_g (ring B)
      if (!mbar_wait(smem_u32(&bars.pa_full), g & 1, abort, 47)) break;
      if (need_o_free && !mbar_wait(smem_u32(&bars.o_free), (items - 1) & 1, abort, 48)) break;
      tc_fence_after();
      mma_accum(tmem + kColA0, tmem + kColS, attn::opaque(dBm + offB(g)), acc_first);
      tc_commit(smem_u32(&bars.b_empty[g % kStB]));                    // dO_g: last reader
      if (!last) {
        // S^T(g + 1) overwrites P^T(g) after dV(g) has read it
        if (!wait_a(gn, 61)) break;
        tc_fence_after();
        issue_s(gn);
      }
      // dK += dS^T (written over dP^T) x Q_g (ring A)
      if (!mbar_wait(smem_u32(&bars.pb_full[0]), g & 1, abort, 63)) break;
      tc_fence_after();
      mma_accum(tmem + kColA1, tmem + kColDP, attn::opaque(dAm + offA(g)), acc_first);
      if (!last) {
        // dP^T(g + 1) overwrites dS^T(g) after dK(g) has read it
        if (!wait_b(gn, 69)) break;
        tc_fence_after();
        issue_dp(gn);
      }
      tc_commit(smem_u32(&bars.a_empty[g % kStA]));                    // Q_g: last reader
    }
    if (last) {
      tc_commit(smem_u32(&bars.fix_empty));
      tc_commit(smem_u32(&bars.o_done));
      ++items;
    }
    head = last;
  }
  tc_commit(smem_u32(&bars.drain));
  mbar_wait(smem_u32(&bars.drain), 0, nullptr, 49);
}

// ---------------------------------------------------------------- softmax warps
// Thread: tile rows r0 = base + lane / 4 and r0 + 8; of every 8-column group k the columns
// 8k + 2c + {0, 1} (register 4k + e: row e < 2 ? r0 : r1, column 8k + 2c + (e & 1)).
// dQ mode: rows are queries (their LSE / D from global), columns keys (>= n_valid masked).
// dK/dV mode: rows are keys (>= n_valid masked), columns queries (LSE / D from the slot).
template <int MODE>
__device__ __forceinline__ void softmax_role(const Args& a, Bars& bars, uint32_t sb, uint32_t tmem, uint32_t warp,
                                             uint32_t lane) {
  using namespace attn;
  volatile int* abort = &bars.abort;
  const uint32_t base = 32 * (warp & 3) + 16 * (warp >> 2);
  const uint32_t lane_off = base << 16;
  const uint32_t r0 = base + lane / 4, c = lane & 3;
  const float sl2 = a.scale * kLog2e;
  const uint64_t c2 = f2_pack(__float_as_uint(sl2), __float_as_uint(sl2));
  uint32_t g = 0, items = 0;
  for (uint32_t ic = 0;; ++ic) {
    const uint32_t is = ic % kItemRec;
    if (!warp_wait_abort(smem_u32(&bars.item_full[is]), (ic / kItemRec) & 1, abort, 55)) break;
    const int32_t ui = reinterpret_cast<volatile int32_t*>(bars.item_u)[is];
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&bars.item_free[is]));
    if (ui < 0) break;
    const int64_t u = ui;
    int32_t nf;
    bool bad;
    const int32_t n = list_len(a, u, nf, bad);
    __nv_bfloat16* o0r0 = a.out0 + (u * 128 + r0) * 128;
    __nv_bfloat16* o0r1 = o0r0 + 8 * 128;
    __nv_bfloat16* o1r0 = MODE == kModeDKDV ? a.out1 + (u * 128 + r0) * 128 : nullptr;
    __nv_bfloat16* o1r1 = MODE == kModeDKDV ? o1r0 + 8 * 128 : nullptr;
    if (n == 0) {
      if (bad && lane == 0 && warp == 0) flag_status(ST_BAD_LIST);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        reinterpret_cast<uint4*>(o0r0 + c * 32)[i] = make_uint4(0, 0, 0, 0);
        reinterpret_cast<uint4*>(o0r1 + c * 32)[i] = make_uint4(0, 0, 0, 0);
        if (MODE == kModeDKDV) {
          reinterpret_cast<uint4*>(o1r0 + c * 32)[i] = make_uint4(0, 0, 0, 0);
          reinterpret_cast<uint4*>(o1r1 + c * 32)[i] = make_uint4(0, 0, 0, 0);
        }
      }
      continue;
    }
    // per-item row statistics (dQ mode) or key-row validity (dK/dV mode)
    uint64_t nl0 = 0, nl1 = 0;   // -LSE log2e of rows r0, r1 (dQ)
    float d0 = 0.f, d1 = 0.f;    // D of rows r0, r1 (dQ)
    bool row0_ok = true, row1_ok = true;
    if (MODE == kModeDQ) {
      const float l0 = -a.lse[u * 128 + r0] * kLog2e, l1 = -a.lse[u * 128 + r0 + 8] * kLog2e;
      nl0 = f2_pack(__float_as_uint(l0), __float_as_uint(l0));
      nl1 = f2_pack(__float_as_uint(l1), __float_as_uint(l1));
      d0 = a.delta[u * 128 + r0];
      d1 = a.delta[u * 128 + r0 + 8];
    } else {
      const int32_t h = static_cast<int32_t>((u / a.nT) % a.H), j = static_cast<int32_t>(u % a.nT);
      const int32_t nvk = a.valid[static_cast<int64_t>(h) * a.nT + j];
      row0_ok = static_cast<int32_t>(r0) < nvk;
      row1_ok = static_cast<int32_t>(r0 + 8) < nvk;
    }
    bool ok = true;
    for (int32_t jj = 0; jj < n; ++jj, ++g) {
      int32_t nv = 128;
      if (MODE == kModeDQ) {
        if (!warp_wait_abort(smem_u32(&bars.rec_full[g % kRec]), (g / kRec) & 1, abort, 50)) { ok = false; break; }
        nv = reinterpret_cast<volatile int32_t*>(bars.rec_nv)[g % kRec];
      }
      if (MODE == kModeDKDV) {
        // the LSE / D rows of the streamed query tile, written by the copy engine
        if (!warp_wait_abort(smem_u32(&bars.st_full[g % kStStat]), (g / kStStat) & 1, abort, 53)) {
          ok = false;
          break;
        }
      }
      // S of this block (dQ: buffer g & 1, one phase per use; dK/dV: one buffer)
      const uint32_t colS = MODE == kModeDQ ? ((g & 1) ? kColS1 : kColS) : kColS;
      if (!warp_wait_abort(smem_u32(&bars.s_full[MODE == kModeDQ ? (g & 1) : 0]),
                           MODE == kModeDQ ? ((g >> 1) & 1) : (g & 1), abort, 51)) { ok = false; break; }
      tc_fence_after();
      uint32_t s[64], dp[64];
      tmem_ld_16x256b_x16(tmem + lane_off + colS, s);
      tmem_wait_ld();
      reg_fence(s);
      if (MODE == kModeDQ) {
        // dP as well, then hand its buffer back so that dP of the next block can be issued
        if (!warp_wait_abort(smem_u32(&bars.dp_full), g & 1, abort, 56)) { ok = false; break; }
        tc_fence_after();
        tmem_ld_16x256b_x16(tmem + lane_off + kColDP, dp);
        tmem_wait_ld();
        reg_fence(dp);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars.dp_free));
      }
      if (MODE == kModeDQ && nv < 128) {
        const int32_t kv0 = (nv - 2 * static_cast<int32_t>(c) + 7) >> 3;
        const int32_t kv1 = (nv - 2 * static_cast<int32_t>(c) + 6) >> 3;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          if (k >= kv0) { s[4 * k] = 0xFF800000u; s[4 * k + 2] = 0xFF800000u; }   // -inf
          if (k >= kv1) { s[4 * k + 1] = 0xFF800000u; s[4 * k + 3] = 0xFF800000u; }
        }
      }
      const uint32_t stat = sb + kOffStat + (g % kStStat) * kStatB;   // dK/dV: LSE, D
      // dQ mode, key tile with at most 64 valid slots: S, dP and dQ's accumulation cover its
      // first 64 keys only; column groups 8..15 are skipped by a warp-uniform branch
      const bool hi = MODE != kModeDQ || nv > 64;
      uint32_t pk[32];
      // P (in place of s), and for dK/dV P^T packed over S
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        if (k == 8 && !hi) break;
        uint64_t na, nb;
        if (MODE == kModeDQ) {
          na = nl0;
          nb = nl1;
        } else {
          // columns are queries: their -LSE log2e, the same for both rows
          float2 l2;
          asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(l2.x), "=f"(l2.y)
                       : "r"(stat + (8 * k + 2 * c) * 4));
          na = f2_pack(__float_as_uint(-l2.x * kLog2e), __float_as_uint(-l2.y * kLog2e));
          nb = na;
        }
        float x0, x1, y0, y1;
        f2_unpack(f2_fma(f2_pack(s[4 * k], s[4 * k + 1]), c2, na), x0, x1);
        f2_unpack(f2_fma(f2_pack(s[4 * k + 2], s[4 * k + 3]), c2, nb), y0, y1);
        float p0 = ex2_approx(x0), p1 = ex2_approx(x1), q0 = ex2_approx(y0), q1 = ex2_approx(y1);
        if (MODE == kModeDKDV) {
          if (!row0_ok) { p0 = 0.f; p1 = 0.f; }
          if (!row1_ok) { q0 = 0.f; q1 = 0.f; }
          pk[2 * k] = pack_bf16x2(p0, p1);
          pk[2 * k + 1] = pack_bf16x2(q0, q1);
        }
        s[4 * k] = __float_as_uint(p0); s[4 * k + 1] = __float_as_uint(p1);
        s[4 * k + 2] = __float_as_uint(q0); s[4 * k + 3] = __float_as_uint(q1);
      }
      if (MODE == kModeDKDV) {
        // P^T over S^T: dV(g) can start while dP^T(g) is still on the tensor core
        tmem_st_16x128b_x16(tmem + lane_off + kColS, pk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars.pa_full));
        if (!warp_wait_abort(smem_u32(&bars.dp_full), g & 1, abort, 57)) { ok = false; break; }
        tc_fence_after();
        tmem_ld_16x256b_x16(tmem + lane_off + kColDP, dp);
        tmem_wait_ld();
        reg_fence(dp);
      }
      // dS = P (dP - D), packed over S (dQ) or over dP (dK/dV)
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        if (k == 8 && !hi) break;
        float da0, da1, db0, db1;
        if (MODE == kModeDQ) {
          da0 = da1 = d0;
          db0 = db1 = d1;
        } else {
          float2 dd;
          asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(dd.x), "=f"(dd.y)
                       : "r"(stat + 512 + (8 * k + 2 * c) * 4));
          da0 = db0 = dd.x;
          da1 = db1 = dd.y;
        }
        const float e0 = __uint_as_float(s[4 * k]) * (__uint_as_float(dp[4 * k]) - da0);
        const float e1 = __uint_as_float(s[4 * k + 1]) * (__uint_as_float(dp[4 * k + 1]) - da1);
        const float f0 = __uint_as_float(s[4 * k + 2]) * (__uint_as_float(dp[4 * k + 2]) - db0);
        const float f1 = __uint_as_float(s[4 * k + 3]) * (__uint_as_float(dp[4 * k + 3]) - db1);
        pk[2 * k] = pack_bf16x2(e0, e1);
        pk[2 * k + 1] = pack_bf16x2(f0, f1);
      }
      if (MODE == kModeDQ) {
        attn::tmem_st_p_half<0>(tmem + lane_off + colS, pk);
        if (hi) attn::tmem_st_p_half<16>(tmem + lane_off + colS + 32, pk);
      } else {
        tmem_st_16x128b_x16(tmem + lane_off + kColDP, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(smem_u32(&bars.pb_full[MODE == kModeDQ ? (g & 1) : 0]));
        if (MODE == kModeDKDV) mbar_arrive(smem_u32(&bars.st_empty[g % kStStat]));   // LSE / D read
      }
    }
    if (!ok) break;
    // epilogue: acc0 (dQ or dV), acc1 (dK) -> bf16 rows; dQ and dK carry the softmax scale
    if (!warp_wait_abort(smem_u32(&bars.o_done), items & 1, abort, 52)) break;
    tc_fence_after();
#pragma unroll 1
    for (int t = 0; t < (MODE == kModeDKDV ? 2 : 1); ++t) {
      const float mul = (MODE == kModeDQ || t == 1) ? a.scale : 1.0f;
      __nv_bfloat16* rA = t == 0 ? o0r0 : o1r0;
      __nv_bfloat16* rB = t == 0 ? o0r1 : o1r1;
      const bool zA = MODE == kModeDKDV && !row0_ok, zB = MODE == kModeDKDV && !row1_ok;   // pad key rows
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t o16[16];
        tmem_ld_16x256b_x4(tmem + lane_off + (t == 0 ? kColA0 : kColA1) + ch * 32, o16);
        tmem_wait_ld();
        reg_fence(o16);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int col = ch * 32 + 8 * q + 2 * static_cast<int>(c);
          *reinterpret_cast<uint32_t*>(rA + col) =
              zA ? 0u : pack_bf16x2(__uint_as_float(o16[4 * q]) * mul, __uint_as_float(o16[4 * q + 1]) * mul);
          *reinterpret_cast<uint32_t*>(rB + col) =
              zB ? 0u : pack_bf16x2(__uint_as_float(o16[4 * q + 2]) * mul, __uint_as_float(o16[4 * q + 3]) * mul);
        }
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&bars.o_free));
    ++items;
  }
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
bwd_kernel(const __grid_constant__ CUtensorMap tmF0, const __grid_constant__ CUtensorMap tmF1,
           const __grid_constant__ CUtensorMap tmS0, const __grid_constant__ CUtensorMap tmS1, const Args a) {
  using namespace attn;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ Bars bars;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const uint32_t tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, wg = warp >> 2;
  volatile int* abort = &bars.abort;
  // the dK/dV instance's shared memory has no alignment slack: it works only from a
  // 1024-byte-aligned start (the same for every thread, so the whole CTA leaves together)
  if (MODE == kModeDKDV && smem != smem_raw) {
    if (tid == 0) flag_status(ST_SMEM_ALIGN);
    return;
  }
  if (tid == 0) {
    mbar_init(smem_u32(&bars.fix_full), 1);
    mbar_init(smem_u32(&bars.fix_empty), 1);
    for (int i = 0; i < kStA; ++i) {
      mbar_init(smem_u32(&bars.a_full[i]), 1);
      mbar_init(smem_u32(&bars.a_empty[i]), 1);
    }
    for (int i = 0; i < kStB; ++i) {
      mbar_init(smem_u32(&bars.b_full[i]), 1);
      mbar_init(smem_u32(&bars.b_empty[i]), 1);
    }
    for (int i = 0; i < kStStat; ++i) {
      mbar_init(smem_u32(&bars.st_full[i]), 1);
      mbar_init(smem_u32(&bars.st_empty[i]), 8);   // the eight softmax warps
    }
    mbar_init(smem_u32(&bars.s_full[0]), 1);
    mbar_init(smem_u32(&bars.s_full[1]), 1);
    mbar_init(smem_u32(&bars.dp_full), 1);
    mbar_init(smem_u32(&bars.dp_free), 8);
    mbar_init(smem_u32(&bars.pa_full), 8);
    mbar_init(smem_u32(&bars.pb_full[0]), 8);
    mbar_init(smem_u32(&bars.pb_full[1]), 8);
    mbar_init(smem_u32(&bars.o_done), 1);
    mbar_init(smem_u32(&bars.o_free), 8);
    mbar_init(smem_u32(&bars.drain), 1);
    for (int i = 0; i < kRec; ++i) mbar_init(smem_u32(&bars.rec_full[i]), 1);
    for (int i = 0; i < kItemRec; ++i) {
      mbar_init(smem_u32(&bars.item_full[i]), 1);
      mbar_init(smem_u32(&bars.item_free[i]), 8);
    }
    bars.abort = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(&bars.tmem_base), kTmemCols);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    prefetch_tensormap(&tmF0);
    prefetch_tensormap(&tmF1);
    prefetch_tensormap(&tmS0);
    prefetch_tensormap(&tmS1);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;
  if (wg == 2) {
    reg_dealloc<kControlRegs>();
    if (warp == 8 && lane == 0)
      role_producer<MODE>(a, bars, sb, &tmF0, &tmF1, &tmS0, &tmS1, abort);
    else if (warp == 9 && lane == 0)
      role_issuer<MODE>(bars, sb, tmem, abort);
  } else {
    reg_alloc<kSoftmaxRegs>();
    softmax_role<MODE>(a, bars, sb, tmem, warp, lane);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9) tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------- D = rowsum(dO * O)
// 16 threads per 256-byte row (16 bytes each), a warp two rows per step.
__global__ void __launch_bounds__(256) delta_kernel(const __nv_bfloat16* __restrict__ dout,
                                                    const __nv_bfloat16* __restrict__ o, float* __restrict__ delta,
                                                    int64_t rows) {
  const uint32_t c = threadIdx.x & 15;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * (blockDim.x / 16);
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 16) + (threadIdx.x >> 4); r < rows; r += stride) {
    const uint4 x = *reinterpret_cast<const uint4*>(dout + r * 128 + c * 8);
    const uint4 y = *reinterpret_cast<const uint4*>(o + r * 128 + c * 8);
    const __nv_bfloat162* xp = reinterpret_cast<const __nv_bfloat162*>(&x);
    const __nv_bfloat162* yp = reinterpret_cast<const __nv_bfloat162*>(&y);
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 a2 = __bfloat1622float2(xp[i]), b2 = __bfloat1622float2(yp[i]);
      acc = fmaf(a2.x, b2.x, acc);
      acc = fmaf(a2.y, b2.y, acc);
    }
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (c == 0) delta[r] = acc;
  }
}

// ---------------------------------------------------------------- transposed lists
// One warp per (b, h, key tile j): for the head's query tiles i in order, a lane tests
// whether j is in row i's ascending full or partial list (binary search); ballot compaction
// writes the hits in ascending i.
__device__ __forceinline__ bool sorted_has(const int32_t* p, int32_t n, int32_t x) {
  int32_t lo = 0, hi = n;
  while (lo < hi) {
    const int32_t mid = (lo + hi) >> 1;
    if (p[mid] < x) lo = mid + 1; else hi = mid;
  }
  return lo < n && p[lo] == x;
}

__global__ void __launch_bounds__(128) transpose_lists_kernel(const int32_t* full_cnt, const int32_t* full_idx,
                                                              const int32_t* part_cnt, const int32_t* part_idx,
                                                              int32_t stride, const int32_t* nT_per_head,
                                                              int32_t* t_cnt, int32_t* t_idx, int32_t t_stride,
                                                              int32_t H, int32_t nT, int64_t rows) {
  const uint32_t lane = threadIdx.x & 31;
  const int64_t u = static_cast<int64_t>(blockIdx.x) * 4 + (threadIdx.x >> 5);
  if (u >= rows) return;
  const int32_t j = static_cast<int32_t>(u % nT), h = static_cast<int32_t>((u / nT) % H);
  int32_t nth = nT_per_head[h];
  if (nth < 0 || nth > nT) {
    if (lane == 0) flag_status(ST_BAD_LIST);
    nth = 0;
  }
  const int64_t row0 = u - j;   // (b, h, 0)
  int32_t cnt = 0;
  uint32_t lt;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(lt));
  for (int32_t i0 = 0; i0 < (j < nth ? nth : 0); i0 += 32) {
    const int32_t i = i0 + static_cast<int32_t>(lane);
    bool hit = false;
    if (i < nth) {
      const int64_t r = row0 + i;
      int32_t nf = full_cnt[r], np = part_cnt[r];
      if (nf < 0 || np < 0 || nf > stride || np > stride) { flag_status(ST_BAD_LIST); nf = 0; np = 0; }
      hit = sorted_has(full_idx + r * stride, nf, j) || sorted_has(part_idx + r * stride, np, j);
    }
    const uint32_t bal = __ballot_sync(0xffffffffu, hit);
    if (hit) {
      const int32_t pos = cnt + __popc(bal & lt);
      if (pos < t_stride) t_idx[u * t_stride + pos] = i;
    }
    cnt += __popc(bal);
  }
  if (lane == 0) {
    if (cnt > t_stride) flag_status(ST_LIST_OVERFLOW);
    t_cnt[u] = cnt < t_stride ? cnt : t_stride;
  }
}

}  // namespace bwd
}  // namespace veda
