// k_attn.cuh -- step 5: block-sparse flash-attention forward on sm_100a.
//
// "Deploying this checkpoint", preamble: attention only visits the selected key
// tiles; section 2 (SM90/SM100): 128 x 128 tiles at head_dim 128 with one 128-row
// query tile per block row, the block mask handed to the kernel as full/partial index
// lists. "Miowtion" README, Key Features: full/partial block lists and a single mask
// function on partial blocks (here: key slots >= n_valid are masked).
//
// One persistent CTA per SM walks (batch, head, query tile) items in head-major order
// (so the CTAs resident at one time share one head's K/V in L2). Per CTA:
//   warps 0..7   softmax: warp w owns the 16 query rows 32 (w % 4) + 16 (w / 4) + [0, 16) of
//                the tile (TMEM lanes; a warp may address the 32-lane window of its w % 4).
//                The 16x256b TMEM shape gives a thread two rows (r, r + 8) and 32 of the 128
//                scores of each; a row's maximum is completed by two shuffles inside the
//                thread quad that shares it, the row sum stays per thread until the epilogue.
//                No warp waits for another warp's data, and all eight run one code path.
//   warp 8       TMA producer of Q (per item) and K_j (kKSt-deep ring); it also writes a
//                record per block (valid key slots) for the softmax
//   warp 11      TMA producer of V_j (kVSt-deep ring), so that a V buffer still in use
//                never holds back the next K load
//   warp 9       Q K^T issuer (one thread): S_b = Q K_j^T, b = block parity, once every
//                softmax warp has taken S(j-2) out of buffer b
//   warp 10      P V issuer (one thread): O += P_b V_j, P_b read from tensor memory
// An eighth of the exponentials (the second row of every fourth column group) run on the FMA
// pipe (exp2_fma_x2) instead of the MUFU. A key tile with at most 64 valid slots (a partial
// tile whose valid prefix fits in half the tile) is computed over its first 64 keys only:
// Q K^T with N = 64, P V with K = 64 and half the softmax, flagged by the producers in the
// ring slot's op word.
// Tensor memory (512 columns): S0 | S1 | O | P0 | P1. With two S buffers, each freed as
// soon as the softmax holds it in registers, and P in buffers of its own, the tensor core
// computes S(j+1) and P V(j-1) while the softmax works on block j. The running maximum (in
// log2 units) is only moved (and O rescaled in TMEM after P V(j-1) has landed) when it grows
// by more than 30, i.e. when P would exceed 2^30; otherwise P uses the stale maximum, exact
// after the division by the row sum.
//
// Every wait is bounded (veda_ptx.cuh): when one runs out the CTA raises a shared abort
// flag, all roles leave their loops, in-flight copies and MMAs are drained with bounded
// waits and the tensor memory is freed before the CTA exits.
#pragma once

#include "veda_ptx.cuh"

namespace veda {
namespace attn {

constexpr int kThreads = 384;
constexpr int kQSt = 2;                    // Q buffers (items)
constexpr int kKSt = 3;                    // K ring (Q K^T issuer)
constexpr int kVSt = 2;                    // V ring (P V issuer)
constexpr int kRec = 8;                    // block records (valid key slots of block g)
static_assert(kRec > kKSt + 2, "a block record is rewritten only after the softmax has read it");
constexpr uint32_t kTileB = 32768;         // 128 x 128 bf16
constexpr uint32_t kHalfB = 16384;         // 128 rows x 64 columns
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kQSt * kTileB;
constexpr uint32_t kOffV = kOffK + kKSt * kTileB;
constexpr uint32_t kSmemTiles = kOffV + kVSt * kTileB;         // 224 KB
constexpr uint32_t kSmemBytes = kSmemTiles + 1024;             // + alignment slack
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256, kColP = 384;         // S_b at 128b, P_b at 384 + 64b
constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 128, 0, 0);   // A, B K-major
constexpr uint32_t kIdescQK64 = idesc_bf16_f32(128, 64, 0, 0);  // the first 64 keys
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 128, 0, 1);   // B (V) MN-major
constexpr float kRescaleLog2 = 30.0f;
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

// One word per K / V ring slot, written by its producer before it arms the slot.
enum : uint32_t {
  kOpNewItem = 1u << 0,   // block 0 of an item (Q K^T: wait for its Q tile; P V: O starts at 0)
  kOpLastBlk = 1u << 1,   // last block of the item
  kOpFirstItem = 1u << 2, // the CTA's first item (no earlier O to wait for)
  kOpStop = 1u << 3,      // end of the stream (no tile)
  kOpHalf = 1u << 4,      // key tile with at most 64 valid slots: Q K^T and P V over keys 0..63
  kOpQBufShift = 8,       // Q buffer of the item (bits 8..)
};

struct Bars {
  uint64_t q_full[kQSt], q_empty[kQSt];
  uint64_t k_full[kKSt], k_empty[kKSt], v_full[kVSt], v_empty[kVSt];
  uint64_t s_full[2], s_free[2], p_full[2], o_done[2];
  uint64_t o_free, drain[2];
  uint64_t rec_full[kRec];
  uint32_t k_op[kKSt], v_op[kVSt];
  int32_t rec_nv[kRec];
  int32_t rec_idx[kRec];
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
// their MMA instead of being hoisted out of the loop into live 64-bit registers.
__device__ __forceinline__ uint64_t opaque(uint64_t x) {
  uint64_t r;
  asm volatile("mov.b64 %0, %1;" : "=l"(r) : "l"(x));
  return r;
}

template <int N>
__device__ __forceinline__ void reg_alloc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void reg_dealloc() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// Valid key slots of block j of an item (entries j >= nf come from the partial list), clamped
// to [1, 128]; the Q / K producer flags out-of-range counts.
__device__ __forceinline__ int32_t block_nv(const int32_t* valid_h, int32_t j, int32_t nf, int32_t idx) {
  if (j < nf) return 128;
  const int32_t nv = valid_h[idx];
  return nv < 1 ? 1 : (nv > 128 ? 128 : nv);
}

// CTA-local item m of the persistent loop.
__device__ __forceinline__ int64_t cta_item(int64_t m) {
  return blockIdx.x + m * static_cast<int64_t>(gridDim.x);
}

// ---------------------------------------------------------------- softmax
// tcgen05 16-lane shapes. 16x256b: thread t of the warp holds, per 8-column group, the
// column pair 2 (t % 4) + {0, 1} of rows t / 4 and t / 4 + 8 (relative to the lane base in
// the address); .xN repeats that for N consecutive 8-column groups. 16x128b: thread t
// holds column t % 4 of the same two rows per 4-column group.
__device__ __forceinline__ void tmem_ld_16x256b_x16(uint32_t taddr, uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, "
      "%35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, "
      "%56, %57, %58, %59, %60, %61, %62, %63}, [%64];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
        "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
        "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
        "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
        "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_16x256b_x4(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x4.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st_16x256b_x4(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x256b.x4.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_st_16x128b_x8(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x128b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_st_16x128b_x16(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x128b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
// P columns 16 OFF / 2 .. + 31 from r[OFF .. OFF + 15] (keys 0..63 for OFF = 0, 64..127 for 16).
template <int OFF>
__device__ __forceinline__ void tmem_st_p_half(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x128b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15, %16};" ::"r"(taddr),
      "r"(r[OFF + 0]), "r"(r[OFF + 1]), "r"(r[OFF + 2]), "r"(r[OFF + 3]), "r"(r[OFF + 4]), "r"(r[OFF + 5]),
      "r"(r[OFF + 6]), "r"(r[OFF + 7]), "r"(r[OFF + 8]), "r"(r[OFF + 9]), "r"(r[OFF + 10]), "r"(r[OFF + 11]),
      "r"(r[OFF + 12]), "r"(r[OFF + 13]), "r"(r[OFF + 14]), "r"(r[OFF + 15])
      : "memory");
}
template <int N>
__device__ __forceinline__ void reg_fence(uint32_t (&r)[N]) {
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
}
__device__ __forceinline__ float quad_max(float v) {
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
  return fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
}
__device__ __forceinline__ float quad_sum(float v) {
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  return v + __shfl_xor_sync(0xffffffffu, v, 2);
}

// One block of one warp's softmax, S in buffer g & 1: takes S into registers and hands the
// buffer back, masks key slots >= nv, computes P with the running maximum (moving it and
// rescaling O when a row's maximum grew by more than 30, in log2 units), adds the row sums
// and hands P over in buffer g & 1. A key tile with at most 64 valid slots had Q K^T and P V
// issued over its first 64 keys only: the softmax then covers column groups 0..7 and skips
// 8..15 by a warp-uniform branch inside the one unrolled loop (a second, narrower copy of the
// loop measured slower: the two copies compete for the instruction cache). Returns false
// when a bounded wait ran out.
__device__ __forceinline__ bool softmax_block(const Args& a, Bars& bars, uint32_t tmem, uint32_t lane_off,
                                              uint32_t c, uint32_t lane, uint32_t g, bool first, int32_t nv,
                                              volatile int* abort, float& m0, float& m1, float& l0, float& l1) {
  const uint32_t sbuf = g & 1;
  tc_fence_after();
  const bool hi = nv > 64;   // the upper 64 keys were computed
  uint32_t s[64];
  tmem_ld_16x256b_x16(tmem + lane_off + kColS + sbuf * 128, s);
  tmem_wait_ld();
  reg_fence(s);
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(smem_u32(&bars.s_free[sbuf]));
  if (nv < 128) {
    // column 8k + 2c + e is a key slot < nv exactly for k < kv_e = ceil((nv - 2c - e) / 8)
    const int32_t kv0 = (nv - 2 * static_cast<int32_t>(c) + 7) >> 3;
    const int32_t kv1 = (nv - 2 * static_cast<int32_t>(c) + 6) >> 3;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      if (k >= kv0) { s[4 * k] = 0xFF800000u; s[4 * k + 2] = 0xFF800000u; }   // -inf
      if (k >= kv1) { s[4 * k + 1] = 0xFF800000u; s[4 * k + 3] = 0xFF800000u; }
    }
  }
  // Exponentials with the current running maximum m, computed together with the block's
  // row maxima (one basic block, so the scheduler interleaves the MUFU and max chains).
  // If a row's maximum (log2 units) grew by more than 30, the reference moves, O is
  // rescaled and the pass is repeated; otherwise P uses the stale maximum, exact after the
  // division by the row sum (P stays below 2^30, far inside bf16 and the fp32 sums of at
  // most nT * 128 terms). Block 0 of an item takes its row maxima first, so that its
  // single pass has a reference.
  if (first) {
    float a4[4], b4[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      a4[q] = fmaxf(__uint_as_float(s[4 * q]), __uint_as_float(s[4 * q + 1]));
      b4[q] = fmaxf(__uint_as_float(s[4 * q + 2]), __uint_as_float(s[4 * q + 3]));
    }
#pragma unroll
    for (int k = 4; k < 16; ++k) {
      if (k == 8 && !hi) break;
      a4[k & 3] = fmax3(a4[k & 3], __uint_as_float(s[4 * k]), __uint_as_float(s[4 * k + 1]));
      b4[k & 3] = fmax3(b4[k & 3], __uint_as_float(s[4 * k + 2]), __uint_as_float(s[4 * k + 3]));
    }
    m0 = quad_max(fmaxf(fmaxf(a4[0], a4[1]), fmaxf(a4[2], a4[3]))) * a.scale_log2;
    m1 = quad_max(fmaxf(fmaxf(b4[0], b4[1]), fmaxf(b4[2], b4[3]))) * a.scale_log2;
  }
  const uint64_t c2 = f2_pack(__float_as_uint(a.scale_log2), __float_as_uint(a.scale_log2));
  uint64_t acc0[2], acc1[2];
  uint32_t pk[32];
#pragma unroll 1
  for (int pass = 0;; ++pass) {
    const uint64_t nm0 = f2_pack(__float_as_uint(-m0), __float_as_uint(-m0));
    const uint64_t nm1 = f2_pack(__float_as_uint(-m1), __float_as_uint(-m1));
    acc0[0] = acc0[1] = acc1[0] = acc1[1] = 0ull;
    float a4[4], b4[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      a4[q] = fmaxf(__uint_as_float(s[4 * q]), __uint_as_float(s[4 * q + 1]));
      b4[q] = fmaxf(__uint_as_float(s[4 * q + 2]), __uint_as_float(s[4 * q + 3]));
    }
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      if (k == 8 && !hi) break;
      if (k >= 4) {
        a4[k & 3] = fmax3(a4[k & 3], __uint_as_float(s[4 * k]), __uint_as_float(s[4 * k + 1]));
        b4[k & 3] = fmax3(b4[k & 3], __uint_as_float(s[4 * k + 2]), __uint_as_float(s[4 * k + 3]));
      }
      float x0, x1, q0, q1;
      f2_unpack(f2_fma(f2_pack(s[4 * k], s[4 * k + 1]), c2, nm0), x0, x1);
      const uint64_t yy = f2_fma(f2_pack(s[4 * k + 2], s[4 * k + 3]), c2, nm1);
      const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
      if ((k & 3) == 3) {   // an eighth of the exponentials on the FMA pipe
        exp2_fma_x2(yy, q0, q1);
      } else {
        float y0, y1;
        f2_unpack(yy, y0, y1);
        q0 = ex2_approx(y0);
        q1 = ex2_approx(y1);
      }
      acc0[k & 1] = f2_add(acc0[k & 1], f2_pack(__float_as_uint(p0), __float_as_uint(p1)));
      acc1[k & 1] = f2_add(acc1[k & 1], f2_pack(__float_as_uint(q0), __float_as_uint(q1)));
      pk[2 * k] = pack_bf16x2(p0, p1);
      pk[2 * k + 1] = pack_bf16x2(q0, q1);
    }
    const float mb0 = quad_max(fmaxf(fmaxf(a4[0], a4[1]), fmaxf(a4[2], a4[3]))) * a.scale_log2;
    const float mb1 = quad_max(fmaxf(fmaxf(b4[0], b4[1]), fmaxf(b4[2], b4[3]))) * a.scale_log2;
    const bool need0 = mb0 > m0 + kRescaleLog2;
    const bool need1 = mb1 > m1 + kRescaleLog2;
    if (pass == 1 || !__any_sync(0xffffffffu, need0 || need1)) break;
    // O must hold P V of every earlier block before it is rescaled
    const uint32_t gp = g - 1;
    if (!warp_wait_abort(smem_u32(&bars.o_done[gp & 1]), (gp >> 1) & 1, abort, 31)) return false;
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
    if (!warp_wait_abort(smem_u32(&bars.o_done[gp & 1]), (gp >> 1) & 1, abort, 32)) return false;
    tc_fence_after();
  }
  tmem_st_p_half<0>(tmem + lane_off + kColP + sbuf * 64, pk);
  if (hi) tmem_st_p_half<16>(tmem + lane_off + kColP + sbuf * 64 + 32, pk);
  tmem_wait_st();
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(smem_u32(&bars.p_full[sbuf]));
  return true;
}

// Softmax and epilogue of one warp's 16 rows for every item of the CTA. Thread (lane)
// holds tile rows r0 = base + lane / 4 and r1 = r0 + 8 and, of every 8-column group k,
// the columns 8k + 2c + {0, 1} (c = lane % 4): register 4k + e is row (e < 2 ? r0 : r1),
// column 8k + 2c + (e & 1).
__device__ __forceinline__ void softmax_role(const Args& a, Bars& bars, uint32_t tmem, uint32_t warp,
                                             uint32_t lane) {
  volatile int* abort = &bars.abort;
  const uint32_t base = 32 * (warp & 3) + 16 * (warp >> 2);   // first TMEM lane (tile row)
  const uint32_t lane_off = base << 16;
  const uint32_t r0 = base + lane / 4, c = lane & 3;
  uint32_t g = 0;
  uint32_t items = 0;
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
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    bool ok = true;
    for (int32_t j = 0; j < n; ++j, ++g) {
      const uint32_t sbuf = g & 1;
      if (!warp_wait_abort(smem_u32(&bars.rec_full[g % kRec]), (g / kRec) & 1, abort, 36)) { ok = false; break; }
      const int32_t nv = reinterpret_cast<volatile int32_t*>(bars.rec_nv)[g % kRec];
      if (!warp_wait_abort(smem_u32(&bars.s_full[sbuf]), (g >> 1) & 1, abort, 30)) { ok = false; break; }
      if (!softmax_block(a, bars, tmem, lane_off, c, lane, g, j == 0, nv, abort, m0, m1, l0, l1)) {
        ok = false;
        break;
      }
    }
    if (!ok) break;
    // epilogue: row sums over the quad, O / l -> bf16, LSE
    const float lt0 = quad_sum(l0), lt1 = quad_sum(l1);
    const uint32_t gl = g - 1;
    if (!warp_wait_abort(smem_u32(&bars.o_done[gl & 1]), (gl >> 1) & 1, abort, 33)) break;
    tc_fence_after();
    const float inv0 = 1.0f / lt0, inv1 = 1.0f / lt1;
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
      a.lse[u * 128 + r0] = (m0 + __log2f(lt0)) * 0.69314718055994531f;
      a.lse[u * 128 + r0 + 8] = (m1 + __log2f(lt1)) * 0.69314718055994531f;
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&bars.o_free));
    ++items;
  }
}

// ---------------------------------------------------------------- control roles
// One thread each. The Q / K producer and the Q K^T issuer are shared with the block-heat
// kernel (k_heat.cuh), which runs the same Q K^T stream without P V.

// TMA producer of Q (per item) and K_j (kKSt-deep ring), plus one record per block (valid
// key slots and key tile index) for the softmax warps.
// kHalfKeys: mark key tiles with at most 64 valid slots (kOpHalf), so that the issuer runs
// Q K^T over their first 64 keys only (the attention; block heat takes whole tiles).
template <bool kHalfKeys>
__device__ __forceinline__ void role_qk_producer(const Args& a, Bars& bars, uint32_t sb, const CUtensorMap* tmQ,
                                                 const CUtensorMap* tmK, volatile int* abort) {
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
    if (qc >= kQSt && !mbar_wait(smem_u32(&bars.q_empty[qb]), (qc / kQSt - 1) & 1, abort, 10)) break;
    const uint32_t qbar = smem_u32(&bars.q_full[qb]);
    mbar_arrive_expect_tx(qbar, kTileB);
    tma_load_2d(sb + kOffQ + qb * kTileB, tmQ, qbar, 0, static_cast<int32_t>(u * 128));
    tma_load_2d(sb + kOffQ + qb * kTileB + kHalfB, tmQ, qbar, 64, static_cast<int32_t>(u * 128));
    const int64_t head_row = (u / a.nT) * a.nT;
    const int32_t* valid_h = a.valid + ((u / a.nT) % a.H) * a.nT;
    for (int32_t j = 0; j < n; ++j) {
      bool b2;
      const int32_t idx = item_key(a, u, nf, j, b2);
      if (b2) flag_status(ST_BAD_LIST);   // clamped to tile 0 by item_key
      const int32_t row = static_cast<int32_t>((head_row + idx) * 128);
      const uint32_t ks = kc % kKSt;
      if (kc >= kKSt && !mbar_wait(smem_u32(&bars.k_empty[ks]), (kc / kKSt - 1) & 1, abort, 11)) { stop = true; break; }
      if (j >= nf && (valid_h[idx] < 1 || valid_h[idx] > 128)) flag_status(ST_BAD_LIST);
      const int32_t nv = block_nv(valid_h, j, nf, idx);
      bars.k_op[ks] = (j == 0 ? kOpNewItem : 0u) | (j == n - 1 ? kOpLastBlk : 0u) |
                      (kHalfKeys && nv <= 64 ? kOpHalf : 0u) | (qb << kOpQBufShift);
      const uint32_t kb = smem_u32(&bars.k_full[ks]);
      mbar_arrive_expect_tx(kb, kTileB);
      tma_load_2d(sb + kOffK + ks * kTileB, tmK, kb, 0, row);
      tma_load_2d(sb + kOffK + ks * kTileB + kHalfB, tmK, kb, 64, row);
      // block record (entry kc % kRec was last read for block kc - kRec, before the
      // softmax freed S(kc - kRec) and so before K(kc - kRec + kKSt + 2) could load)
      bars.rec_nv[kc % kRec] = nv;
      bars.rec_idx[kc % kRec] = idx;
      mbar_arrive(smem_u32(&bars.rec_full[kc % kRec]));
      ++kc;
    }
    ++qc;
  }
  if (!*abort) {
    // end of stream: one more K slot carrying only the stop record
    const uint32_t ks = kc % kKSt;
    if (kc < kKSt || mbar_wait(smem_u32(&bars.k_empty[ks]), (kc / kKSt - 1) & 1, abort, 16)) {
      bars.k_op[ks] = kOpStop;
      mbar_arrive(smem_u32(&bars.k_full[ks]));
    }
  }
  if (*abort) {
    // let the copies this thread issued land before the CTA exits
    for (uint32_t i = kc > kKSt ? kc - kKSt : 0; i < kc; ++i)
      mbar_wait(smem_u32(&bars.k_full[i % kKSt]), (i / kKSt) & 1, nullptr, 13);
    for (uint32_t i = qc > kQSt ? qc - kQSt : 0; i < qc; ++i)
      mbar_wait(smem_u32(&bars.q_full[i % kQSt]), (i / kQSt) & 1, nullptr, 14);
  }
}

// TMA producer of V_j (kVSt-deep ring).
__device__ __forceinline__ void role_v_producer(const Args& a, Bars& bars, uint32_t sb, const CUtensorMap* tmV,
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
    const int32_t* valid_h = a.valid + ((u / a.nT) % a.H) * a.nT;
    for (int32_t j = 0; j < n; ++j) {
      bool b2;
      const int32_t idx = item_key(a, u, nf, j, b2);
      const int32_t row = static_cast<int32_t>((head_row + idx) * 128);
      const uint32_t vs = vc % kVSt;
      if (vc >= kVSt && !mbar_wait(smem_u32(&bars.v_empty[vs]), (vc / kVSt - 1) & 1, abort, 12)) { stop = true; break; }
      bars.v_op[vs] = (j == 0 ? kOpNewItem : 0u) | (j == n - 1 ? kOpLastBlk : 0u) | (items == 0 ? kOpFirstItem : 0u) |
                      (block_nv(valid_h, j, nf, idx) <= 64 ? kOpHalf : 0u);
      const uint32_t vb = smem_u32(&bars.v_full[vs]);
      mbar_arrive_expect_tx(vb, kTileB);
      tma_load_2d(sb + kOffV + vs * kTileB, tmV, vb, 0, row);
      tma_load_2d(sb + kOffV + vs * kTileB + kHalfB, tmV, vb, 64, row);
      ++vc;
    }
    ++items;
  }
  if (!*abort) {
    const uint32_t vs = vc % kVSt;
    if (vc < kVSt || mbar_wait(smem_u32(&bars.v_empty[vs]), (vc / kVSt - 1) & 1, abort, 17)) {
      bars.v_op[vs] = kOpStop;
      mbar_arrive(smem_u32(&bars.v_full[vs]));
    }
  }
  if (*abort) {
    for (uint32_t i = vc > kVSt ? vc - kVSt : 0; i < vc; ++i)
      mbar_wait(smem_u32(&bars.v_full[i % kVSt]), (i / kVSt) & 1, nullptr, 18);
  }
}

// Q K^T issuer: S_b = Q K_j^T into TMEM buffer b = j & 1 once every softmax warp has taken
// S(j - 2) out of it.
__device__ __forceinline__ void role_qk_issuer(Bars& bars, uint32_t sb, uint32_t tmem, volatile int* abort) {
  // S buffer b = g & 1 is free once every softmax warp holds S(g - 2) in registers.
  // Descriptors of the tile bases; a k-step or another ring slot only moves the 14-bit
  // start-address field (16-byte units), which never carries for addresses < 256 KB.
  const uint64_t dQ = smem_desc_sw128(sb + kOffQ, 16, 1024);
  const uint64_t dK = smem_desc_sw128(sb + kOffK, 16, 1024);
  uint32_t qn[kQSt];
  for (int i = 0; i < kQSt; ++i) qn[i] = 0;   // Q tiles consumed per buffer
  for (uint32_t g = 0;; ++g) {
    const uint32_t ks = g % kKSt;
    if (!mbar_wait(smem_u32(&bars.k_full[ks]), (g / kKSt) & 1, abort, 23)) break;
    const uint32_t op = bars.k_op[ks];
    if (op & kOpStop) break;
    const uint32_t qb = op >> kOpQBufShift;
    if (op & kOpNewItem) {
      if (!mbar_wait(smem_u32(&bars.q_full[qb]), qn[qb] & 1, abort, 20)) break;
      ++qn[qb];
    }
    const uint32_t sbuf = g & 1;
    if (g >= 2 && !mbar_wait(smem_u32(&bars.s_free[sbuf]), ((g >> 1) - 1) & 1, abort, 26)) break;
    tc_fence_after();
    const uint64_t a0 = opaque(dQ + static_cast<uint64_t>(qb * (kTileB >> 4)));
    const uint64_t b0 = opaque(dK + static_cast<uint64_t>(ks * (kTileB >> 4)));
    const uint32_t d = tmem + kColS + sbuf * 128;
    const uint32_t idesc = (op & kOpHalf) ? kIdescQK64 : kIdescQK;   // N = 64: keys 0..63
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const uint64_t koff = static_cast<uint64_t>((kk >> 2) * (kHalfB >> 4) + (kk & 3) * 2);
      mma_ss(d, a0 + koff, b0 + koff, idesc, kk > 0 ? 1u : 0u);
    }
    tc_commit(smem_u32(&bars.s_full[sbuf]));
    if (op & kOpLastBlk) tc_commit(smem_u32(&bars.q_empty[qb]));
    tc_commit(smem_u32(&bars.k_empty[ks]));
  }
  tc_commit(smem_u32(&bars.drain[0]));
  mbar_wait(smem_u32(&bars.drain[0]), 0, nullptr, 25);
}

// P V issuer: O += P_b V_j with P_b read from TMEM.
__device__ __forceinline__ void role_pv_issuer(Bars& bars, uint32_t sb, uint32_t tmem, volatile int* abort) {
  const uint64_t dV = smem_desc_sw128(sb + kOffV, kHalfB, 1024);
  uint32_t items_done = 0;
  for (uint32_t g = 0;; ++g) {
    const uint32_t vs = g % kVSt;
    if (!mbar_wait(smem_u32(&bars.v_full[vs]), (g / kVSt) & 1, abort, 24)) break;
    const uint32_t op = bars.v_op[vs];
    if (op & kOpStop) break;
    const uint32_t pb = g & 1;
    if (!mbar_wait(smem_u32(&bars.p_full[pb]), (g >> 1) & 1, abort, 21)) break;
    // the first P V of an item overwrites O: the previous item's epilogue must be done
    if ((op & kOpNewItem) && !(op & kOpFirstItem) &&
        !mbar_wait(smem_u32(&bars.o_free), (items_done - 1) & 1, abort, 22))
      break;
    tc_fence_after();
    const uint64_t b0 = opaque(dV + static_cast<uint64_t>(vs * (kTileB >> 4)));
    const uint32_t pa = tmem + kColP + pb * 64;
    mma_ts(tmem + kColO, pa, b0, kIdescPV, (op & kOpNewItem) ? 0u : 1u);
#pragma unroll
    for (int kk = 1; kk < 4; ++kk)
      mma_ts(tmem + kColO, pa + kk * 8, b0 + static_cast<uint64_t>(kk * (2048 >> 4)), kIdescPV, 1u);
    if (!(op & kOpHalf)) {   // keys 64..127 (P columns 32..63, V rows 64..127)
#pragma unroll
      for (int kk = 4; kk < 8; ++kk)
        mma_ts(tmem + kColO, pa + kk * 8, b0 + static_cast<uint64_t>(kk * (2048 >> 4)), kIdescPV, 1u);
    }
    tc_commit(smem_u32(&bars.o_done[pb]));
    tc_commit(smem_u32(&bars.v_empty[vs]));
    if (op & kOpLastBlk) ++items_done;
  }
  tc_commit(smem_u32(&bars.drain[1]));
  mbar_wait(smem_u32(&bars.drain[1]), 0, nullptr, 27);
}

// Barrier setup of a CTA (thread 0).
__device__ __forceinline__ void init_bars(Bars& bars) {
  for (int i = 0; i < kQSt; ++i) {
    mbar_init(smem_u32(&bars.q_full[i]), 1);
    mbar_init(smem_u32(&bars.q_empty[i]), 1);
  }
  for (int i = 0; i < kKSt; ++i) {
    mbar_init(smem_u32(&bars.k_full[i]), 1);
    mbar_init(smem_u32(&bars.k_empty[i]), 1);
  }
  for (int i = 0; i < kVSt; ++i) {
    mbar_init(smem_u32(&bars.v_full[i]), 1);
    mbar_init(smem_u32(&bars.v_empty[i]), 1);
  }
  for (int i = 0; i < 2; ++i) {
    mbar_init(smem_u32(&bars.s_full[i]), 1);
    mbar_init(smem_u32(&bars.s_free[i]), 8);
    mbar_init(smem_u32(&bars.p_full[i]), 8);
    mbar_init(smem_u32(&bars.o_done[i]), 1);
    mbar_init(smem_u32(&bars.drain[i]), 1);
  }
  for (int i = 0; i < kRec; ++i) mbar_init(smem_u32(&bars.rec_full[i]), 1);
  mbar_init(smem_u32(&bars.o_free), 8);
  bars.abort = 0;
  fence_mbar_init();
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

  if (tid == 0) init_bars(bars);
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
    if (warp == 8 && lane == 0)
      role_qk_producer<true>(a, bars, sb, &tmQ, &tmK, abort);
    else if (warp == 11 && lane == 0)
      role_v_producer(a, bars, sb, &tmV, abort);
    else if (warp == 9 && lane == 0)
      role_qk_issuer(bars, sb, tmem, abort);
    else if (warp == 10 && lane == 0)
      role_pv_issuer(bars, sb, tmem, abort);
  } else {
    reg_alloc<kSoftmaxRegs>();
    softmax_role(a, bars, tmem, warp, lane);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace attn
}  // namespace veda
