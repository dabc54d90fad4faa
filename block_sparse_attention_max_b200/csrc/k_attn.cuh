// k_attn.cuh -- step 5: block-sparse flash-attention forward on sm_100a.
//
// "Deploying this checkpoint", preamble: attention only visits the selected key
// tiles; section 2 (SM90/SM100): 128 x 128 tiles at head_dim 128 with one 128-row
// query tile per block row, the block mask handed to the kernel as full/partial index
// lists. "Miowtion" README, Key Features: full/partial block lists and a single mask
// function on partial blocks (here: key slots >= n_valid are masked).
//
// One persistent CTA per SM walks (batch, head, query tile) items in head-major order
// (so the CTAs resident at one time share one head's K/V in L2). Roles:
//   warp 4     TMA producer: Q tile, then K_j / V_j of the listed key tiles (128B swizzle)
//   warp 5     MMA issuer (one thread): S = Q K^T into tensor memory (tcgen05, M=N=128,
//              bf16 in, fp32 out), O += P V with P read from tensor memory
//   warps 0-3  softmax + epilogue, one query row per thread (the 32x32b TMEM access
//              shape gives each thread a whole row, so the row max and sum need no shuffle)
// Tensor memory (512 columns): S0 | S1 | O | P0 | P1. Two S and P buffers let the MMA
// compute S_{j+1} and P_{j-1} V_{j-1} while the softmax works on S_j. The running
// maximum is only moved (and O rescaled in TMEM) when it grows by more than 2^8;
// otherwise P is computed against the stale maximum, which is exact after the final
// division by the row sum.
//
// Every wait is bounded (veda_ptx.cuh): when one runs out the CTA raises a shared abort
// flag, all roles leave their loops, in-flight copies and MMAs are drained with bounded
// waits and the tensor memory is freed before the CTA exits.
#pragma once

#include "veda_ptx.cuh"

namespace veda {
namespace attn {

constexpr int kThreads = 192;
constexpr int kKStages = 3;
constexpr int kVStages = 2;
constexpr uint32_t kTileB = 32768;   // 128 x 128 bf16
constexpr uint32_t kHalfB = 16384;   // 128 rows x 64 columns
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + kTileB;
constexpr uint32_t kOffV = kOffK + kKStages * kTileB;
constexpr uint32_t kSmemTiles = kOffV + kVStages * kTileB;   // 192 KB
constexpr uint32_t kSmemBytes = kSmemTiles + 1024;           // + alignment slack
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256, kColP = 384;       // S_b at b*128, P_b at 384 + b*64
constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 128, 0, 0);   // A, B K-major
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 128, 0, 1);   // B (V) MN-major
constexpr float kRescaleLog2 = 8.0f;

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

struct Bars {
  uint64_t q_full, q_empty;
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t v_full[kVStages], v_empty[kVStages];
  uint64_t s_full[2], p_full[2], o_done[2];
  uint64_t o_free, drain;
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

// Whole-warp bounded wait: lane 0 waits, the verdict is shared, and every lane then
// observes the completed phase itself.
__device__ __forceinline__ bool warp_wait_abort(uint32_t bar, uint32_t parity, volatile int* abort,
                                                uint32_t site) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abort, site);
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (ok) ok = mbar_try_wait(bar, parity);
  return __all_sync(0xffffffffu, ok);
}

__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const Args a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ Bars bars;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const uint32_t tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  volatile int* abort = &bars.abort;

  if (tid == 0) {
    mbar_init(smem_u32(&bars.q_full), 1);
    mbar_init(smem_u32(&bars.q_empty), 1);
    for (int i = 0; i < kKStages; ++i) {
      mbar_init(smem_u32(&bars.k_full[i]), 1);
      mbar_init(smem_u32(&bars.k_empty[i]), 1);
    }
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(smem_u32(&bars.v_full[i]), 1);
      mbar_init(smem_u32(&bars.v_empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bars.s_full[i]), 1);
      mbar_init(smem_u32(&bars.p_full[i]), 4);
      mbar_init(smem_u32(&bars.o_done[i]), 1);
    }
    mbar_init(smem_u32(&bars.o_free), 4);
    mbar_init(smem_u32(&bars.drain), 1);
    bars.abort = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(&bars.tmem_base), kTmemCols);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    prefetch_tensormap(&tmQ);
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t kc = 0, vc = 0, qc = 0;
      bool stop = false;
      for (int64_t u = blockIdx.x; u < a.items && !stop; u += gridDim.x) {
        int32_t nf;
        bool bad;
        const int32_t n = item_blocks(a, u, nf, bad);
        if (n == 0) continue;
        const int64_t bh = u / a.nT;
        if (qc > 0 && !mbar_wait(smem_u32(&bars.q_empty), (qc - 1) & 1, abort, 10)) break;
        mbar_arrive_expect_tx(smem_u32(&bars.q_full), kTileB);
        tma_load_2d(sb + kOffQ, &tmQ, smem_u32(&bars.q_full), 0, static_cast<int32_t>(u * 128));
        tma_load_2d(sb + kOffQ + kHalfB, &tmQ, smem_u32(&bars.q_full), 64, static_cast<int32_t>(u * 128));
        ++qc;
        auto load_k = [&](int32_t j) -> bool {
          const uint32_t st = kc % kKStages;
          if (kc >= kKStages && !mbar_wait(smem_u32(&bars.k_empty[st]), (kc / kKStages - 1) & 1, abort, 11))
            return false;
          bool b2;
          const int32_t idx = item_key(a, u, nf, j, b2);
          if (b2) flag_status(ST_BAD_LIST);   // clamped to tile 0 by item_key
          const int32_t row = static_cast<int32_t>((bh * a.nT + idx) * 128);
          const uint32_t bar = smem_u32(&bars.k_full[st]);
          mbar_arrive_expect_tx(bar, kTileB);
          tma_load_2d(sb + kOffK + st * kTileB, &tmK, bar, 0, row);
          tma_load_2d(sb + kOffK + st * kTileB + kHalfB, &tmK, bar, 64, row);
          ++kc;
          return true;
        };
        auto load_v = [&](int32_t j) -> bool {
          const uint32_t st = vc % kVStages;
          if (vc >= kVStages && !mbar_wait(smem_u32(&bars.v_empty[st]), (vc / kVStages - 1) & 1, abort, 12))
            return false;
          bool b2;
          const int32_t idx = item_key(a, u, nf, j, b2);
          const int32_t row = static_cast<int32_t>((bh * a.nT + idx) * 128);
          const uint32_t bar = smem_u32(&bars.v_full[st]);
          mbar_arrive_expect_tx(bar, kTileB);
          tma_load_2d(sb + kOffV + st * kTileB, &tmV, bar, 0, row);
          tma_load_2d(sb + kOffV + st * kTileB + kHalfB, &tmV, bar, 64, row);
          ++vc;
          return true;
        };
        for (int32_t j = 0; j < n && !stop; ++j) {
          if (!load_k(j)) { stop = true; break; }
          if (j >= 1 && !load_v(j - 1)) { stop = true; break; }
        }
        if (!stop && !load_v(n - 1)) stop = true;
      }
      if (*abort) {
        // let the copies this thread issued land before the CTA exits
        for (uint32_t i = kc > kKStages ? kc - kKStages : 0; i < kc; ++i)
          mbar_wait(smem_u32(&bars.k_full[i % kKStages]), (i / kKStages) & 1, nullptr, 13);
        for (uint32_t i = vc > kVStages ? vc - kVStages : 0; i < vc; ++i)
          mbar_wait(smem_u32(&bars.v_full[i % kVStages]), (i / kVStages) & 1, nullptr, 14);
        if (qc > 0) mbar_wait(smem_u32(&bars.q_full), (qc - 1) & 1, nullptr, 15);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t kc = 0, vc = 0, qc = 0, g = 0;
      bool stop = false;
      auto pv = [&](uint32_t gp, bool first) -> bool {
        const uint32_t pb = gp & 1;
        if (!mbar_wait(smem_u32(&bars.p_full[pb]), (gp >> 1) & 1, abort, 20)) return false;
        const uint32_t vs = vc % kVStages;
        if (!mbar_wait(smem_u32(&bars.v_full[vs]), (vc / kVStages) & 1, abort, 21)) return false;
        if (first && qc >= 2 && !mbar_wait(smem_u32(&bars.o_free), (qc - 2) & 1, abort, 22)) return false;
        tc_fence_after();
        const uint32_t vt = sb + kOffV + vs * kTileB;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tmem + kColO, tmem + kColP + pb * 64 + kk * 8, desc_mnmajor(vt, kk), kIdescPV,
                 (first && kk == 0) ? 0u : 1u);
        tc_commit(smem_u32(&bars.o_done[pb]));
        tc_commit(smem_u32(&bars.v_empty[vs]));
        ++vc;
        return true;
      };
      for (int64_t u = blockIdx.x; u < a.items && !stop; u += gridDim.x) {
        int32_t nf;
        bool bad;
        const int32_t n = item_blocks(a, u, nf, bad);
        if (n == 0) continue;
        if (!mbar_wait(smem_u32(&bars.q_full), qc & 1, abort, 23)) break;
        ++qc;
        tc_fence_after();
        for (int32_t j = 0; j < n; ++j) {
          const uint32_t st = kc % kKStages;
          if (!mbar_wait(smem_u32(&bars.k_full[st]), (kc / kKStages) & 1, abort, 24)) { stop = true; break; }
          tc_fence_after();
          const uint32_t kt = sb + kOffK + st * kTileB;
          const uint32_t sbuf = g & 1;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss(tmem + kColS + sbuf * 128, desc_kmajor(sb + kOffQ, kk), desc_kmajor(kt, kk), kIdescQK,
                   kk > 0 ? 1u : 0u);
          tc_commit(smem_u32(&bars.s_full[sbuf]));
          tc_commit(smem_u32(&bars.k_empty[st]));
          ++kc;
          if (j == n - 1) tc_commit(smem_u32(&bars.q_empty));
          if (j >= 1 && !pv(g - 1, j == 1)) { stop = true; break; }
          ++g;
        }
        if (stop) break;
        if (!pv(g - 1, n == 1)) break;
      }
      // drain: every MMA issued so far completes before the tensor memory is freed
      tc_commit(smem_u32(&bars.drain));
      mbar_wait(smem_u32(&bars.drain), 0, nullptr, 25);
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const uint32_t row = tid;                                  // 0..127 = TMEM lane
    const uint32_t lane_off = (warp * 32u) << 16;
    uint32_t g = 0;
    bool stop = false;
    for (int64_t u = blockIdx.x; u < a.items && !stop; u += gridDim.x) {
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
        const uint32_t sbuf = g & 1;
        if (!warp_wait_abort(smem_u32(&bars.s_full[sbuf]), (g >> 1) & 1, abort, 30)) { stop = true; break; }
        tc_fence_after();
        float s[128];
        {
          // four 32-column loads in flight, one wait
          uint32_t r0[32], r1[32], r2[32], r3[32];
          const uint32_t sa = tmem + lane_off + kColS + sbuf * 128;
          tmem_ld32(sa, r0);
          tmem_ld32(sa + 32, r1);
          tmem_ld32(sa + 64, r2);
          tmem_ld32(sa + 96, r3);
          tmem_wait_ld();
          reg_fence32(r0); reg_fence32(r1); reg_fence32(r2); reg_fence32(r3);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            s[i] = __uint_as_float(r0[i]);
            s[32 + i] = __uint_as_float(r1[i]);
            s[64 + i] = __uint_as_float(r2[i]);
            s[96 + i] = __uint_as_float(r3[i]);
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
            if (i >= nv) s[i] = -INFINITY;
        }
        // row max with eight independent chains (a single chain is 128 dependent steps)
        float mx8[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) mx8[c] = s[c];
#pragma unroll
        for (int i = 8; i < 128; ++i) mx8[i & 7] = fmaxf(mx8[i & 7], s[i]);
        const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                               fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
        const float m_blk = mx * a.scale_log2;
        if (j == 0) {
          m = m_blk;
        } else {
          const bool need = m_blk > m + kRescaleLog2;
          if (__any_sync(0xffffffffu, need)) {
            // O must hold P V of every earlier block before it is rescaled
            const uint32_t gp = g - 1;
            if (!warp_wait_abort(smem_u32(&bars.o_done[gp & 1]), (gp >> 1) & 1, abort, 31)) { stop = true; break; }
            tc_fence_after();
            const float alpha = need ? ex2_approx(m - m_blk) : 1.0f;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint32_t r32[32];
              tmem_ld32_sync(tmem + lane_off + kColO + c * 32, r32);
#pragma unroll
              for (int i = 0; i < 32; ++i) r32[i] = __float_as_uint(__uint_as_float(r32[i]) * alpha);
              tmem_st32(tmem + lane_off + kColO + c * 32, r32);
            }
            tmem_wait_st();
            if (need) { l *= alpha; m = m_blk; }
          }
        }
        // P_b is free once P_{g-2} V_{g-2} has completed
        if (g >= 2) {
          const uint32_t gp = g - 2;
          if (!warp_wait_abort(smem_u32(&bars.o_done[gp & 1]), (gp >> 1) & 1, abort, 32)) { stop = true; break; }
          tc_fence_after();
        }
        float rs8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < 128; ++i) {
          s[i] = ex2_approx(fmaf(s[i], a.scale_log2, -m));
          rs8[i & 7] += s[i];
        }
        l += ((rs8[0] + rs8[1]) + (rs8[2] + rs8[3])) + ((rs8[4] + rs8[5]) + (rs8[6] + rs8[7]));
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t p32[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) p32[i] = pack_bf16x2(s[c * 64 + 2 * i], s[c * 64 + 2 * i + 1]);
          tmem_st32(tmem + lane_off + kColP + sbuf * 64 + c * 32, p32);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars.p_full[sbuf]));
        ++g;
      }
      if (stop) break;
      if (list_bad && row == 0) flag_status(ST_BAD_LIST);
      // epilogue: O / l -> bf16 rows, LSE
      const uint32_t gl = g - 1;
      if (!warp_wait_abort(smem_u32(&bars.o_done[gl & 1]), (gl >> 1) & 1, abort, 33)) break;
      tc_fence_after();
      const float inv_l = 1.0f / l;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r32[32];
        tmem_ld32_sync(tmem + lane_off + kColO + c * 32, r32);
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
      if (lane == 0) mbar_arrive(smem_u32(&bars.o_free));
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace attn
}  // namespace veda
