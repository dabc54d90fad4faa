// k_attn.cuh -- step 5: block-sparse flash-attention forward on sm_100a.
//
// "Deploying this checkpoint", preamble: attention only visits the selected key
// tiles; section 2 (SM90/SM100): 128 x 128 tiles at head_dim 128 with one 128-row
// query tile per block row, the block mask handed to the kernel as full/partial index
// lists. "Miowtion" README, Key Features: full/partial block lists and a single mask
// function on partial blocks (here: key slots >= n_valid are masked).
//
// One persistent CTA per SM walks (batch, head, query tile) items in head-major order
// (so the CTAs resident at one time share one head's K/V in L2). A CTA works on two
// query tiles at once ("slots" 0 and 1), so that while one slot's softmax runs the
// tensor core works for the other:
//   warpgroup 0 / 1   softmax + epilogue of slot 0 / 1, one query row per thread (the
//                     32x32b TMEM access shape gives each thread a whole row, so the row
//                     max and sum need no shuffle)
//   warp 8            TMA producer: Q of each slot's item, then the K or V tile every MMA
//                     op needs, in MMA order, through one 5-slot ring (128B swizzle)
//   warp 9            MMA issuer (one thread, tcgen05.mma kind::f16, M = N = 128):
//                     S_i = Q_i K^T (shared-memory operands, K-major) and
//                     O_i += P_i V (P_i read from tensor memory, V MN-major)
// Tensor memory: slot i owns columns [256 i, 256 i + 256): S_i in the first 128, O_i in
// the next 128; P_i (bf16 pairs) is written over the first 64 columns of S_i once S_i
// has been read. Per slot the MMA order is QK(0), PV(0), QK(1), PV(1), ...; tcgen05 MMAs
// from one thread execute in issue order, so QK(j+1) overwrites S_i only after PV(j) has
// read P_i. The two slots' streams are merged as QK0(0), QK1(0), PV0(0), QK0(1),
// PV1(0), QK1(1), PV0(1), ...; the producer replays the same stream to fill the ring.
// The running maximum is only moved (and O rescaled in place) when it grows by more
// than 2^8; otherwise P uses the stale maximum, exact after the division by the row
// sum. O_i is stable when S_i(j) is signalled: the commit that signals S_i(j) also
// covers P_i(j-1) V.
//
// Every wait is bounded (veda_ptx.cuh): when one runs out the CTA raises a shared abort
// flag, all roles leave their loops, in-flight copies and MMAs are drained with bounded
// waits and the tensor memory is freed before the CTA exits.
#pragma once

#include "veda_ptx.cuh"

namespace veda {
namespace attn {

constexpr int kThreads = 384;
constexpr int kStages = 5;                 // K/V ring
constexpr uint32_t kTileB = 32768;         // 128 x 128 bf16
constexpr uint32_t kHalfB = 16384;         // 128 rows x 64 columns
constexpr uint32_t kOffQ = 0;              // Q_0, Q_1
constexpr uint32_t kOffRing = 2 * kTileB;
constexpr uint32_t kSmemTiles = kOffRing + kStages * kTileB;   // 224 KB
constexpr uint32_t kSmemBytes = kSmemTiles + 1024;             // + alignment slack
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 128, 0, 0);   // A, B K-major
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 128, 0, 1);   // B (V) MN-major
constexpr float kRescaleLog2 = 8.0f;
// register split (setmaxnreg): two softmax warpgroups and one producer/MMA warpgroup;
// the total equals the block's allocation at launch (384 threads x 168 registers)
constexpr int kLaunchRegs = 168;
constexpr int kSoftmaxRegs = 224;
constexpr int kControlRegs = 56;
static_assert(2 * kSoftmaxRegs + kControlRegs <= 3 * kLaunchRegs, "register split exceeds the launch");

struct Args {
  const int32_t* valid;      // [H][nT]
  const int32_t* full_cnt;   // [B*H*nT]
  const int32_t* full_idx;   // [B*H*nT][stride]
  const int32_t* part_cnt;
  const int32_t* part_idx;
  __nv_bfloat16* o;          // [B*H*nT*128][128]
  float* lse;                // [B*H*nT*128] or null
  int32_t stride, H, nT;
  int64_t items;             // B*H*nT
  float scale_log2;          // softmax scale * log2(e)
};

// One word per ring slot, written by the producer before it arms the slot: what the MMA
// issuer has to do with the tile.
enum : uint32_t {
  kOpPV = 1u << 0,        // P V (else Q K^T)
  kOpNewItem = 1u << 1,   // Q K^T of a slot's new item: wait for its Q tile
  kOpFirstBlk = 1u << 2,  // block 0 of the item (P V overwrites O)
  kOpLastBlk = 1u << 3,   // last block of the item
  kOpSlot1 = 1u << 4,     // slot 1 (else slot 0)
  kOpFirstItem = 1u << 5, // the slot's first item (no earlier O to wait for)
  kOpStop = 1u << 6,      // end of the stream (no tile)
};

struct Bars {
  uint64_t full[kStages], empty[kStages];
  uint32_t op[kStages];
  uint64_t q_full[2], q_empty[2];
  uint64_t s_full[2], p_full[2], o_done[2], o_free[2];
  uint64_t drain;
  uint32_t tmem_base;
  int32_t abort;
};

// Block count of an item and a check that its lists are well formed (every role reads
// the same memory, so every role reaches the same verdict).
__device__ __forceinline__ int32_t item_blocks(const Args& a, int64_t u, int32_t& nf, bool& bad) {
  nf = a.full_cnt[u];
  const int32_t np = a.part_cnt[u];
  bad = nf < 0 || np < 0 || nf > a.stride || np > a.stride || nf + np > a.nT;
  if (bad) { nf = 0; return 0; }
  return nf + np;
}
__device__ __forceinline__ int32_t item_key(const Args& a, int64_t u, int32_t nf, int32_t j,
                                            bool& bad) {
  int32_t idx = j < nf ? a.full_idx[u * a.stride + j] : a.part_idx[u * a.stride + (j - nf)];
  bad = idx < 0 || idx >= a.nT;
  return bad ? 0 : idx;
}

// K-major operand (Q or K tile): k-step kk covers columns [16kk, 16kk+16).
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t tile, int kk) {
  return smem_desc_sw128(tile + (kk >> 2) * kHalfB + (kk & 3) * 32, 16, 1024);
}
// MN-major operand (V tile as B of P V): k-step kk covers keys [16kk, 16kk+16);
// the two 64-column halves are LBO = 16 KB apart, 8-key groups SBO = 1 KB apart.
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t tile, int kk) {
  return smem_desc_sw128(tile + kk * 2048, kHalfB, 1024);
}

// Whole-warp bounded wait: every lane polls the barrier and the warp leaves together
// (a completed phase stays completed until the warp consumes it, so once one lane sees
// it, all lanes do on their next poll). Fast path: one try_wait and one vote.
__device__ __forceinline__ bool warp_wait_abort(uint32_t bar, uint32_t parity, volatile int* abort,
                                                uint32_t site) {
  if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
    if ((it & 31u) == 0) {
      int give_up = 0;
      if ((threadIdx.x & 31) == 0) {
        if (*abort) {
          give_up = 1;
        } else if (globaltimer_ns() - t0 > kWaitLimitNs) {
          flag_status(ST_TIMEOUT | ((site & 0xffu) << ST_WAIT_SITE_SHIFT));
          *abort = 1;
          give_up = 1;
        }
      }
      if (__shfl_sync(0xffffffffu, give_up, 0)) return false;
    }
  }
}

template <int N>
__device__ __forceinline__ void reg_alloc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void reg_dealloc() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// ------------------------------------------------------------------------------------
// The merged MMA op stream of the two slots (replayed identically by producer and MMA).
// Slot i takes the CTA's items m = i, i + 2, i + 4, ... (item u = blockIdx.x + m * grid)
// that have at least one listed key tile.
// ------------------------------------------------------------------------------------
struct Op {
  int32_t slot, j, n, nf;
  int64_t u;
  bool pv;         // P V (else Q K^T)
  bool new_item;   // Q K^T of a slot's new item (needs its Q tile)
  bool first_item; // the slot's first item (no earlier O to wait for)
};

struct Stream {
  int64_t m[2];     // CTA-local item index of each slot's current item
  int64_t u[2];
  int32_t n[2], nf[2], j[2];
  bool live[2], started[2];
  int32_t slot_turn;   // slot whose unit comes next
  int32_t pending_qk;  // after a slot's PV, its QK is emitted next (-1 if none)
  int32_t init;        // initial QKs still to emit (2 .. 0)
  int32_t items_done[2];

  __device__ void seek(const Args& a, int s, int64_t from) {
    live[s] = false;
    for (int64_t mm = from;; mm += 2) {
      const int64_t uu = blockIdx.x + mm * static_cast<int64_t>(gridDim.x);
      if (uu >= a.items) return;
      bool bad;
      int32_t f;
      const int32_t nn = item_blocks(a, uu, f, bad);
      if (nn > 0) {
        m[s] = mm; u[s] = uu; n[s] = nn; nf[s] = f; j[s] = 0; live[s] = true;
        return;
      }
    }
  }
  __device__ void start(const Args& a) {
    seek(a, 0, 0);
    seek(a, 1, 1);
    items_done[0] = items_done[1] = 0;
    slot_turn = 0;
    pending_qk = -1;
    init = 0;
  }
  __device__ Op qk_op(int s, bool fresh) const {
    Op o;
    o.slot = s; o.j = j[s]; o.n = n[s]; o.nf = nf[s]; o.u = u[s]; o.pv = false;
    o.new_item = fresh; o.first_item = items_done[s] == 0;
    return o;
  }
  // Next op; false when both slots are done.
  __device__ bool next(const Args& a, Op& o) {
    if (init < 2) {                         // QK0(0), QK1(0)
      while (init < 2) {
        const int s = init++;
        if (live[s]) { o = qk_op(s, true); return true; }
      }
    }
    if (pending_qk >= 0) {                  // the QK that follows a slot's PV
      const int s = pending_qk;
      pending_qk = -1;
      o = qk_op(s, j[s] == 0);
      return true;
    }
    for (int t = 0; t < 2; ++t) {
      const int s = (slot_turn + t) & 1;
      if (!live[s]) continue;
      slot_turn = s ^ 1;
      o.slot = s; o.j = j[s]; o.n = n[s]; o.nf = nf[s]; o.u = u[s]; o.pv = true;
      o.new_item = false; o.first_item = items_done[s] == 0;
      if (j[s] + 1 < n[s]) {
        ++j[s];
      } else {
        ++items_done[s];
        seek(a, s, m[s] + 2);
      }
      if (live[s]) pending_qk = s;
      return true;
    }
    return false;
  }
};

__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const Args a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ Bars bars;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const uint32_t tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, wg = warp >> 2;
  volatile int* abort = &bars.abort;

  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(smem_u32(&bars.full[i]), 1);
      mbar_init(smem_u32(&bars.empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bars.q_full[i]), 1);
      mbar_init(smem_u32(&bars.q_empty[i]), 1);
      mbar_init(smem_u32(&bars.s_full[i]), 1);
      mbar_init(smem_u32(&bars.p_full[i]), 4);
      mbar_init(smem_u32(&bars.o_done[i]), 1);
      mbar_init(smem_u32(&bars.o_free[i]), 4);
    }
    mbar_init(smem_u32(&bars.drain), 1);
    bars.abort = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(&bars.tmem_base), kTmemCols);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    prefetch_tensormap(&tmQ);
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;

  if (wg == 2) {
    reg_dealloc<kControlRegs>();
    if (warp == 8 && lane == 0) {
      // ---------------------------------------------------------- TMA producer
      Stream st;
      st.start(a);
      uint32_t lc = 0;           // ring loads issued
      uint32_t qc[2] = {0, 0};   // Q loads issued per slot
      Op o;
      while (st.next(a, o)) {
        const int s = o.slot;
        if (o.new_item) {
          if (qc[s] > 0 && !mbar_wait(smem_u32(&bars.q_empty[s]), (qc[s] - 1) & 1, abort, 10)) break;
          const uint32_t qb = smem_u32(&bars.q_full[s]);
          mbar_arrive_expect_tx(qb, kTileB);
          tma_load_2d(sb + kOffQ + s * kTileB, &tmQ, qb, 0, static_cast<int32_t>(o.u * 128));
          tma_load_2d(sb + kOffQ + s * kTileB + kHalfB, &tmQ, qb, 64, static_cast<int32_t>(o.u * 128));
          ++qc[s];
        }
        const uint32_t stg = lc % kStages;
        if (lc >= kStages && !mbar_wait(smem_u32(&bars.empty[stg]), (lc / kStages - 1) & 1, abort, 11)) break;
        bool bad;
        const int32_t idx = item_key(a, o.u, o.nf, o.j, bad);
        if (bad) flag_status(ST_BAD_LIST);
        const int32_t row = static_cast<int32_t>(((o.u / a.nT) * a.nT + idx) * 128);
        const uint32_t fb = smem_u32(&bars.full[stg]);
        const CUtensorMap* map = o.pv ? &tmV : &tmK;
        bars.op[stg] = (o.pv ? kOpPV : 0u) | (o.new_item ? kOpNewItem : 0u) | (o.j == 0 ? kOpFirstBlk : 0u) |
                       (o.j == o.n - 1 ? kOpLastBlk : 0u) | (s ? kOpSlot1 : 0u) | (o.first_item ? kOpFirstItem : 0u);
        mbar_arrive_expect_tx(fb, kTileB);
        tma_load_2d(sb + kOffRing + stg * kTileB, map, fb, 0, row);
        tma_load_2d(sb + kOffRing + stg * kTileB + kHalfB, map, fb, 64, row);
        ++lc;
      }
      if (!*abort) {
        // end of stream: one more ring slot carrying only the stop record
        const uint32_t stg = lc % kStages;
        if (lc < kStages || mbar_wait(smem_u32(&bars.empty[stg]), (lc / kStages - 1) & 1, abort, 12)) {
          bars.op[stg] = kOpStop;
          mbar_arrive(smem_u32(&bars.full[stg]));
        }
      }
      if (*abort) {
        // let the copies this thread issued land before the CTA exits
        for (uint32_t i = lc > kStages ? lc - kStages : 0; i < lc; ++i)
          mbar_wait(smem_u32(&bars.full[i % kStages]), (i / kStages) & 1, nullptr, 13);
        for (int s = 0; s < 2; ++s)
          if (qc[s] > 0) mbar_wait(smem_u32(&bars.q_full[s]), (qc[s] - 1) & 1, nullptr, 14);
      }
    } else if (warp == 9 && lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      // Consumes the ring in order; each slot's op record says what to issue. No stream
      // bookkeeping here: between two ops the tensor pipe only has ~1 MMA queued, so the
      // issuer must get from one op's last MMA to the next op's first in a few dozen cycles.
      // Descriptors of the tile bases; a k-step or another ring slot only moves the 14-bit
      // start-address field (16-byte units), which never carries for addresses < 256 KB.
      const uint64_t dQ = smem_desc_sw128(sb + kOffQ, 16, 1024);          // Q_0 (K-major)
      const uint64_t dK = smem_desc_sw128(sb + kOffRing, 16, 1024);       // ring slot 0 as K
      const uint64_t dV = smem_desc_sw128(sb + kOffRing, kHalfB, 1024);   // ring slot 0 as V
      uint32_t qc0 = 0, qc1 = 0, pc0 = 0, pc1 = 0, oc0 = 0, oc1 = 0;
      for (uint32_t lc = 0;; ++lc) {
        const uint32_t stg = lc % kStages;
        if (!mbar_wait(smem_u32(&bars.full[stg]), (lc / kStages) & 1, abort, 23)) break;
        const uint32_t op = bars.op[stg];
        if (op & kOpStop) break;
        const uint32_t s = (op & kOpSlot1) ? 1u : 0u;
        const uint32_t s_col = tmem + s * 256, o_col = s_col + 128;
        const uint64_t ring_off = static_cast<uint64_t>(stg * (kTileB >> 4));
        if (!(op & kOpPV)) {
          if (op & kOpNewItem) {
            uint32_t& qc = s ? qc1 : qc0;
            if (!mbar_wait(smem_u32(&bars.q_full[s]), qc & 1, abort, 20)) break;
            ++qc;
          }
          tc_fence_after();
          const uint64_t a0 = dQ + static_cast<uint64_t>(s * (kTileB >> 4));
          const uint64_t b0 = dK + ring_off;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t koff = static_cast<uint64_t>((kk >> 2) * (kHalfB >> 4) + (kk & 3) * 2);
            mma_ss(s_col, a0 + koff, b0 + koff, kIdescQK, kk > 0 ? 1u : 0u);
          }
          tc_commit(smem_u32(&bars.s_full[s]));
          if (op & kOpLastBlk) tc_commit(smem_u32(&bars.q_empty[s]));
        } else {
          uint32_t& pc = s ? pc1 : pc0;
          if (!mbar_wait(smem_u32(&bars.p_full[s]), pc & 1, abort, 21)) break;
          ++pc;
          // the first P V of an item overwrites O_i: the previous item's epilogue must be done
          if ((op & kOpFirstBlk) && !(op & kOpFirstItem)) {
            const uint32_t oc = s ? oc1 : oc0;
            if (!mbar_wait(smem_u32(&bars.o_free[s]), (oc - 1) & 1, abort, 22)) break;
          }
          tc_fence_after();
          const uint64_t b0 = dV + ring_off;
          mma_ts(o_col, s_col, b0, kIdescPV, (op & kOpFirstBlk) ? 0u : 1u);
#pragma unroll
          for (int kk = 1; kk < 8; ++kk)
            mma_ts(o_col, s_col + kk * 8, b0 + static_cast<uint64_t>(kk * (2048 >> 4)), kIdescPV, 1u);
          if (op & kOpLastBlk) {
            tc_commit(smem_u32(&bars.o_done[s]));
            if (s) ++oc1; else ++oc0;
          }
        }
        tc_commit(smem_u32(&bars.empty[stg]));
      }
      // drain: every MMA issued so far completes before the tensor memory is freed
      tc_commit(smem_u32(&bars.drain));
      mbar_wait(smem_u32(&bars.drain), 0, nullptr, 25);
    }
  } else {
    reg_alloc<kSoftmaxRegs>();
    // ------------------------------------------------------------ softmax + epilogue
    const int slot = static_cast<int>(wg);
    const uint32_t row = tid & 127;                              // TMEM lane
    const uint32_t lane_off = ((warp & 3) * 32u) << 16;
    const uint32_t s_col = tmem + lane_off + slot * 256, o_col = s_col + 128;
    uint32_t sc = 0, ic = 0;      // S tiles consumed, items finished (this slot)
    bool stop = false;
    for (int64_t mm = slot;; mm += 2) {
      const int64_t u = blockIdx.x + mm * static_cast<int64_t>(gridDim.x);
      if (u >= a.items || stop) break;
      int32_t nf;
      bool bad;
      const int32_t n = item_blocks(a, u, nf, bad);
      const int64_t grow = u * 128 + row;
      uint4* orow = reinterpret_cast<uint4*>(a.o + grow * 128);
      if (n == 0) {
        if (bad && row == 0) flag_status(ST_BAD_LIST);
#pragma unroll
        for (int c = 0; c < 16; ++c) orow[c] = make_uint4(0, 0, 0, 0);
        if (a.lse) a.lse[grow] = -INFINITY;
        continue;
      }
      const int32_t h = static_cast<int32_t>((u / a.nT) % a.H);
      float m = -INFINITY, l = 0.f;
      bool list_bad = false;
      for (int32_t j = 0; j < n; ++j) {
        if (!warp_wait_abort(smem_u32(&bars.s_full[slot]), sc & 1, abort, 30)) { stop = true; break; }
        ++sc;
        tc_fence_after();
        uint32_t s[128];   // raw fp32 bits of this row of S
        {
          uint32_t r0[32], r1[32], r2[32], r3[32];
          tmem_ld32(s_col, r0);
          tmem_ld32(s_col + 32, r1);
          tmem_ld32(s_col + 64, r2);
          tmem_ld32(s_col + 96, r3);
          tmem_wait_ld();
          reg_fence32(r0); reg_fence32(r1); reg_fence32(r2); reg_fence32(r3);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            s[i] = r0[i]; s[32 + i] = r1[i]; s[64 + i] = r2[i]; s[96 + i] = r3[i];
          }
        }
        int32_t nv = 128;
        if (j >= nf) {
          bool b2;
          const int32_t idx = item_key(a, u, nf, j, b2);
          list_bad |= b2;
          nv = a.valid[static_cast<int64_t>(h) * a.nT + idx];
          if (nv < 1 || nv > 128) { list_bad = true; nv = nv < 1 ? 1 : 128; }
        }
        if (nv < 128) {
#pragma unroll
          for (int i = 0; i < 128; ++i)
            if (i >= nv) s[i] = 0xFF800000u;   // -inf
        }
        // row max: eight independent chains of 3-input max
        float mx8[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) mx8[c] = __uint_as_float(s[c]);
#pragma unroll
        for (int i = 8; i < 128; i += 2)
          mx8[(i >> 1) & 7] = fmax3(mx8[(i >> 1) & 7], __uint_as_float(s[i]), __uint_as_float(s[i + 1]));
        const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                               fmaxf(mx8[6], mx8[7]));
        const float m_blk = mx * a.scale_log2;
        if (j == 0) {
          m = m_blk;
        } else {
          const bool need = m_blk > m + kRescaleLog2;
          if (__any_sync(0xffffffffu, need)) {
            // O_i already holds P V of every earlier block (covered by the S commit)
            const float alpha = need ? ex2_approx(m - m_blk) : 1.0f;
            const uint64_t alpha2 = f2_pack(__float_as_uint(alpha), __float_as_uint(alpha));
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint32_t r32[32];
              tmem_ld32_sync(o_col + c * 32, r32);
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const uint64_t v = f2_mul(f2_pack(r32[2 * i], r32[2 * i + 1]), alpha2);
                float lo, hi;
                f2_unpack(v, lo, hi);
                r32[2 * i] = __float_as_uint(lo);
                r32[2 * i + 1] = __float_as_uint(hi);
              }
              tmem_st32(o_col + c * 32, r32);
            }
            tmem_wait_st();
            if (need) { l *= alpha; m = m_blk; }
          }
        }
        // p = 2^(s * scale_log2 - m): scale-and-subtract and the row sum in fp32 pairs
        const uint64_t c2 = f2_pack(__float_as_uint(a.scale_log2), __float_as_uint(a.scale_log2));
        const uint64_t nm2 = f2_pack(__float_as_uint(-m), __float_as_uint(-m));
        uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
        uint32_t pk[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(s[2 * i], s[2 * i + 1]), c2, nm2), x0, x1);
          const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
          acc[i & 3] = f2_add(acc[i & 3], f2_pack(__float_as_uint(p0), __float_as_uint(p1)));
          pk[i] = pack_bf16x2(p0, p1);
        }
        {
          float t0, t1, t2, t3, t4, t5, t6, t7;
          f2_unpack(acc[0], t0, t1); f2_unpack(acc[1], t2, t3);
          f2_unpack(acc[2], t4, t5); f2_unpack(acc[3], t6, t7);
          l += ((t0 + t1) + (t2 + t3)) + ((t4 + t5) + (t6 + t7));
        }
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t p32[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) p32[i] = pk[c * 32 + i];
          tmem_st32(s_col + c * 32, p32);   // P over the first 64 columns of S
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars.p_full[slot]));
      }
      if (stop) break;
      if (list_bad && row == 0) flag_status(ST_BAD_LIST);
      // epilogue: O / l -> bf16 rows, LSE
      if (!warp_wait_abort(smem_u32(&bars.o_done[slot]), ic & 1, abort, 33)) break;
      ++ic;
      tc_fence_after();
      const float inv_l = 1.0f / l;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r32[32];
        tmem_ld32_sync(o_col + c * 32, r32);
        uint32_t packed[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          packed[i] = pack_bf16x2(__uint_as_float(r32[2 * i]) * inv_l, __uint_as_float(r32[2 * i + 1]) * inv_l);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          orow[c * 4 + i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
      }
      if (a.lse) a.lse[grow] = (m + __log2f(l)) * 0.69314718055994531f;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars.o_free[slot]));
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace attn
}  // namespace veda
