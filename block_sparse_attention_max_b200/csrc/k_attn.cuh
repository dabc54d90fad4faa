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
//   warps 8 / 11      TMA producer of slot 0 / 1: the slot's Q tile per item and its K_j,
//                     V_j tiles into the slot's own buffers (128B swizzle)
//   warps 9 / 10      MMA issuer of slot 0 / 1 (one thread each, tcgen05.mma kind::f16,
//                     M = N = 128): S_i = Q_i K^T (shared-memory operands, K-major) and
//                     O_i += P_i V (P_i read from tensor memory, V MN-major). With one
//                     issuer per slot, a slot waiting for its softmax never holds up the
//                     other slot's MMAs.
// Tensor memory: slot i owns columns [256 i, 256 i + 256): S_i in the first 128, O_i in
// the next 128; P_i (bf16 pairs) is written over the first 64 columns of S_i once S_i
// has been read. Per slot the MMA order is QK(0), PV(0), QK(1), PV(1), ...; tcgen05 MMAs
// from one thread execute in issue order, so QK(j+1) overwrites S_i only after PV(j) has
// read P_i, and QK(j+1) is issued right behind PV(j).
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
constexpr int kKSt = 1;                    // K buffers per slot
constexpr int kVSt = 1;                    // V buffers per slot
constexpr int kRec = 8;                    // block records per slot (valid keys of block j)
constexpr uint32_t kTileB = 32768;         // 128 x 128 bf16
constexpr uint32_t kHalfB = 16384;         // 128 rows x 64 columns
constexpr uint32_t kSlotB = (1 + kKSt + kVSt) * kTileB;        // Q, K ring, V ring of a slot
constexpr uint32_t kOffK = kTileB, kOffV = kTileB * (1 + kKSt); // offsets within a slot
constexpr uint32_t kSmemTiles = 2 * kSlotB;                    // 192 KB
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

// One word per K buffer, written by the slot's producer before it arms the buffer: what
// the slot's issuer does with block j (Q K^T now, P V once the softmax is done).
enum : uint32_t {
  kOpNewItem = 1u << 0,   // block 0 of an item: wait for its Q tile; P V overwrites O
  kOpLastBlk = 1u << 1,   // last block of the item
  kOpFirstItem = 1u << 2, // the slot's first item (no earlier O to wait for)
  kOpStop = 1u << 3,      // end of the slot's stream (no tile)
};

struct SlotBars {
  uint64_t k_full[kKSt], k_empty[kKSt], v_full[kVSt], v_empty[kVSt];
  uint64_t q_full, q_empty, s_full, p_full, o_done, o_free, drain;
  uint32_t k_op[kKSt];
  // block records: the producer writes the number of valid key slots of the slot's block
  // b into rec_nv[b % kRec] and arrives on rec_full[b % kRec]; it reuses an entry only
  // after its K buffer came back, i.e. after the softmax finished block b - 2 >= b - kRec
  uint64_t rec_full[kRec];
  int32_t rec_nv[kRec];
};

struct Bars {
  SlotBars sl[2];
  // turn taking of the two softmax warpgroups' exponential phases: group i waits on
  // turn[i], and each of its warps arrives on turn[i ^ 1] when its exponentials are
  // done; a group that has finished all its items raises finished[i] and arrives once
  // more, after which the other group runs alone
  uint64_t turn[2];
  int32_t finished[2];
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

// Hides a value from the optimizer, so that per-k-step descriptors are formed next to
// their MMA instead of being hoisted out of the loop into 24 live 64-bit registers.
__device__ __forceinline__ uint64_t opaque(uint64_t x) {
  uint64_t r;
  asm volatile("mov.b64 %0, %1;" : "=l"(r) : "l"(x));
  return r;
}

// Bounded wait for a softmax group's turn: the turn barrier's phase, or the other group
// having finished all its work.
__device__ __forceinline__ bool turn_wait(uint32_t bar, uint32_t parity, volatile int32_t* other_finished,
                                          volatile int* abort, uint32_t site) {
  if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
    int give_up = 0, done = 0;
    if ((threadIdx.x & 31) == 0) {
      done = *other_finished != 0;
      if (!done && (it & 31u) == 0) {
        if (*abort) {
          give_up = 1;
        } else if (globaltimer_ns() - t0 > kWaitLimitNs) {
          flag_status(ST_TIMEOUT | ((site & 0xffu) << ST_WAIT_SITE_SHIFT));
          *abort = 1;
          give_up = 1;
        }
      }
    }
    done = __shfl_sync(0xffffffffu, done, 0);
    if (done) return true;
    if (__shfl_sync(0xffffffffu, give_up, 0)) return false;
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

// CTA-local item m of the persistent loop: slot i takes m = i, i + 2, i + 4, ...
__device__ __forceinline__ int64_t cta_item(int64_t m) {
  return blockIdx.x + m * static_cast<int64_t>(gridDim.x);
}

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
    for (int i = 0; i < 2; ++i) {
      SlotBars& b = bars.sl[i];
      for (int k = 0; k < kKSt; ++k) {
        mbar_init(smem_u32(&b.k_full[k]), 1);
        mbar_init(smem_u32(&b.k_empty[k]), 1);
      }
      for (int k = 0; k < kVSt; ++k) {
        mbar_init(smem_u32(&b.v_full[k]), 1);
        mbar_init(smem_u32(&b.v_empty[k]), 1);
      }
      mbar_init(smem_u32(&b.q_full), 1);
      mbar_init(smem_u32(&b.q_empty), 1);
      mbar_init(smem_u32(&b.s_full), 1);
      mbar_init(smem_u32(&b.p_full), 4);
      mbar_init(smem_u32(&b.o_done), 1);
      mbar_init(smem_u32(&b.o_free), 4);
      mbar_init(smem_u32(&b.drain), 1);
      for (int k = 0; k < kRec; ++k) mbar_init(smem_u32(&b.rec_full[k]), 1);
      mbar_init(smem_u32(&bars.turn[i]), 4);
      bars.finished[i] = 0;
    }
    bars.abort = 0;
    fence_mbar_init();
  }
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
    reg_dealloc<kControlRegs>();
    if ((warp == 8 || warp == 11) && lane == 0) {
      // ---------------------------------------------------------- TMA producer of a slot
      const int sl = warp == 8 ? 0 : 1;
      SlotBars& b = bars.sl[sl];
      const uint32_t base = sb + sl * kSlotB;
      uint32_t kc = 0, vc = 0, qc = 0;
      bool stop = false;
      for (int64_t mm = sl; !stop; mm += 2) {
        const int64_t u = cta_item(mm);
        if (u >= a.items) break;
        int32_t nf;
        bool bad;
        const int32_t n = item_blocks(a, u, nf, bad);
        if (n == 0) continue;
        if (qc > 0 && !mbar_wait(smem_u32(&b.q_empty), (qc - 1) & 1, abort, 10)) break;
        mbar_arrive_expect_tx(smem_u32(&b.q_full), kTileB);
        tma_load_2d(base, &tmQ, smem_u32(&b.q_full), 0, static_cast<int32_t>(u * 128));
        tma_load_2d(base + kHalfB, &tmQ, smem_u32(&b.q_full), 64, static_cast<int32_t>(u * 128));
        const int64_t head_row = (u / a.nT) * a.nT;
        const int32_t* valid_h = a.valid + ((u / a.nT) % a.H) * a.nT;
        for (int32_t j = 0; j < n; ++j) {
          bool b2;
          const int32_t idx = item_key(a, u, nf, j, b2);
          if (b2) flag_status(ST_BAD_LIST);   // clamped to tile 0 by item_key
          const int32_t row = static_cast<int32_t>((head_row + idx) * 128);
          const uint32_t ks = kc % kKSt;
          if (kc >= kKSt && !mbar_wait(smem_u32(&b.k_empty[ks]), (kc / kKSt - 1) & 1, abort, 11)) { stop = true; break; }
          b.k_op[ks] = (j == 0 ? kOpNewItem : 0u) | (j == n - 1 ? kOpLastBlk : 0u) | (qc == 0 ? kOpFirstItem : 0u);
          const uint32_t kb = smem_u32(&b.k_full[ks]);
          mbar_arrive_expect_tx(kb, kTileB);
          tma_load_2d(base + kOffK + ks * kTileB, &tmK, kb, 0, row);
          tma_load_2d(base + kOffK + ks * kTileB + kHalfB, &tmK, kb, 64, row);
          // the block's record (entry kc % kRec was last read for block kc - kRec <= kc - 2)
          int32_t nv = 128;
          if (j >= nf) {
            nv = valid_h[idx];
            if (nv < 1 || nv > 128) {
              flag_status(ST_BAD_LIST);
              nv = nv < 1 ? 1 : 128;
            }
          }
          b.rec_nv[kc % kRec] = nv;
          mbar_arrive(smem_u32(&b.rec_full[kc % kRec]));
          ++kc;
          const uint32_t vs = vc % kVSt;
          if (vc >= kVSt && !mbar_wait(smem_u32(&b.v_empty[vs]), (vc / kVSt - 1) & 1, abort, 12)) { stop = true; break; }
          const uint32_t vb = smem_u32(&b.v_full[vs]);
          mbar_arrive_expect_tx(vb, kTileB);
          tma_load_2d(base + kOffV + vs * kTileB, &tmV, vb, 0, row);
          tma_load_2d(base + kOffV + vs * kTileB + kHalfB, &tmV, vb, 64, row);
          ++vc;
        }
        ++qc;
      }
      if (!*abort) {
        // end of the slot's stream: one more K buffer carrying only the stop record
        const uint32_t ks = kc % kKSt;
        if (kc < kKSt || mbar_wait(smem_u32(&b.k_empty[ks]), (kc / kKSt - 1) & 1, abort, 16)) {
          b.k_op[ks] = kOpStop;
          mbar_arrive(smem_u32(&b.k_full[ks]));
        }
      }
      if (*abort) {
        // let the copies this thread issued land before the CTA exits
        for (uint32_t i = kc > kKSt ? kc - kKSt : 0; i < kc; ++i)
          mbar_wait(smem_u32(&b.k_full[i % kKSt]), (i / kKSt) & 1, nullptr, 13);
        for (uint32_t i = vc > kVSt ? vc - kVSt : 0; i < vc; ++i)
          mbar_wait(smem_u32(&b.v_full[i % kVSt]), (i / kVSt) & 1, nullptr, 18);
        if (qc > 0) mbar_wait(smem_u32(&b.q_full), (qc - 1) & 1, nullptr, 14);
      }
    } else if ((warp == 9 || warp == 10) && lane == 0) {
      // ---------------------------------------------------------- MMA issuer of a slot
      // Per block j: Q K^T into S_i as soon as K_j is in, then P V once the softmax has
      // written P_i(j). Descriptors of the tile bases; a k-step or another buffer only moves
      // the 14-bit start-address field (16-byte units), which never carries below 256 KB.
      const int sl = warp - 9;
      SlotBars& b = bars.sl[sl];
      const uint32_t base = sb + sl * kSlotB;
      const uint64_t dQ = smem_desc_sw128(base, 16, 1024);
      const uint64_t dK = smem_desc_sw128(base + kOffK, 16, 1024);
      const uint64_t dV = smem_desc_sw128(base + kOffV, kHalfB, 1024);
      const uint32_t s_col = tmem + sl * 256, o_col = s_col + 128;
      uint32_t qc = 0, pc = 0, oc = 0, vc = 0;
      for (uint32_t kc = 0;; ++kc) {
        const uint32_t ks = kc % kKSt;
        if (!mbar_wait(smem_u32(&b.k_full[ks]), (kc / kKSt) & 1, abort, 23)) break;
        const uint32_t op = b.k_op[ks];
        if (op & kOpStop) break;
        if (op & kOpNewItem) {
          if (!mbar_wait(smem_u32(&b.q_full), qc & 1, abort, 20)) break;
          ++qc;
        }
        tc_fence_after();
        const uint64_t a0 = opaque(dQ);
        const uint64_t b0 = opaque(dK + static_cast<uint64_t>(ks * (kTileB >> 4)));
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t koff = static_cast<uint64_t>((kk >> 2) * (kHalfB >> 4) + (kk & 3) * 2);
          mma_ss(s_col, a0 + koff, b0 + koff, kIdescQK, kk > 0 ? 1u : 0u);
        }
        tc_commit(smem_u32(&b.s_full));
        if (op & kOpLastBlk) tc_commit(smem_u32(&b.q_empty));
        tc_commit(smem_u32(&b.k_empty[ks]));
        // P V of the same block
        if (!mbar_wait(smem_u32(&b.p_full), pc & 1, abort, 21)) break;
        ++pc;
        const uint32_t vs = vc % kVSt;
        if (!mbar_wait(smem_u32(&b.v_full[vs]), (vc / kVSt) & 1, abort, 24)) break;
        // the first P V of an item overwrites O_i: the previous item's epilogue must be done
        if ((op & kOpNewItem) && !(op & kOpFirstItem) && !mbar_wait(smem_u32(&b.o_free), (oc - 1) & 1, abort, 22))
          break;
        tc_fence_after();
        const uint64_t v0 = opaque(dV + static_cast<uint64_t>(vs * (kTileB >> 4)));
        mma_ts(o_col, s_col, v0, kIdescPV, (op & kOpNewItem) ? 0u : 1u);
#pragma unroll
        for (int kk = 1; kk < 8; ++kk)
          mma_ts(o_col, s_col + kk * 8, v0 + static_cast<uint64_t>(kk * (2048 >> 4)), kIdescPV, 1u);
        tc_commit(smem_u32(&b.v_empty[vs]));
        ++vc;
        if (op & kOpLastBlk) {
          tc_commit(smem_u32(&b.o_done));
          ++oc;
        }
      }
      // drain: every MMA issued so far completes before the tensor memory is freed
      tc_commit(smem_u32(&b.drain));
      mbar_wait(smem_u32(&b.drain), 0, nullptr, 25);
    }
  } else {
    reg_alloc<kSoftmaxRegs>();
    // ------------------------------------------------------------ softmax + epilogue
    const int slot = static_cast<int>(wg);
    const uint32_t row = tid & 127;                              // TMEM lane
    const uint32_t lane_off = ((warp & 3) * 32u) << 16;
    const uint32_t s_col = tmem + lane_off + slot * 256, o_col = s_col + 128;
    SlotBars& b = bars.sl[slot];
    uint32_t sc = 0, ic = 0;      // S tiles consumed, items finished (this slot)
    uint32_t tc = 0;              // exponential turns taken
    bool stop = false;
    volatile int32_t* other_finished = &bars.finished[slot ^ 1];
    if (slot == 1) {
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars.turn[0]));   // group 0 goes first
    }
    for (int64_t mm = slot;; mm += 2) {
      const int64_t u = cta_item(mm);
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
      for (int32_t j = 0; j < n; ++j) {
        if (!warp_wait_abort(smem_u32(&b.rec_full[sc % kRec]), (sc / kRec) & 1, abort, 34)) { stop = true; break; }
        int32_t nv = reinterpret_cast<volatile int32_t*>(b.rec_nv)[sc % kRec];
        if (!warp_wait_abort(smem_u32(&b.s_full), sc & 1, abort, 30)) { stop = true; break; }
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
        // this group's turn for the exponentials (the other group works on its load, max
        // and P store meanwhile)
        if (!turn_wait(smem_u32(&bars.turn[slot]), tc & 1, other_finished, abort, 35)) { stop = true; break; }
        ++tc;
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
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars.turn[slot ^ 1]));
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
        if (lane == 0) mbar_arrive(smem_u32(&b.p_full));
      }
      if (stop) break;
      // epilogue: O / l -> bf16 rows, LSE
      if (!warp_wait_abort(smem_u32(&b.o_done), ic & 1, abort, 33)) break;
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
      if (lane == 0) mbar_arrive(smem_u32(&b.o_free));
    }
    // this group is done: the other one no longer waits for turns
    __syncwarp();
    if (lane == 0) {
      reinterpret_cast<volatile int32_t*>(&bars.finished[slot])[0] = 1;
      __threadfence_block();
      mbar_arrive(smem_u32(&bars.turn[slot ^ 1]));
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace attn
}  // namespace veda
