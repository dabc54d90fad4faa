// k_scores.cuh -- step 3: per-head residual projection of the pooled features and the
// (query tile, key tile) score matrix, on the tcgen05 tensor cores.
//
// "Miowtion" README, bullet "Sparse acceleration (Veda)" (a small per-head predictor
// scores (query tile, key tile) pairs) and Key Features ("mean/max/min pooling +
// per-head residual projection"):
//   qhat = mean_q + Wq[h] [mean; max; min]_q,   khat likewise,   S = qhat khat^T.
// Both products are "NT" GEMMs, C[M][N] = A[M][K] B[N][K]^T with K contiguous in both
// operands: the projection (M = nT, N = 128, K = 384, plus the mean as residual) and the
// scores (M = N = nT, K = 128).
//
// The scores must agree with the fp64 definition to ~1e-3 relative, beyond what one tf32
// (or bf16) product gives, so every product runs as three tf32 products of a split
// operand (the "3xTF32" scheme): x = hi(x) + lo(x) with hi(x) = tf32(x) and
// lo(x) = tf32(x - hi(x)), and
//   A B^T ~= hi(A) hi(B)^T + hi(A) lo(B)^T + lo(A) hi(B)^T,
// whose dropped term lo(A) lo(B)^T and the rounding of lo are ~2^-21 of |A||B| -- far
// below the tolerance -- while every product runs at the tensor-core tf32 rate with an
// fp32 accumulator in tensor memory.
//
// Kernel: persistent, one CTA per SM, one 128 x 128 output tile at a time.
//   warp 8       TMA producer: per 32-deep K chunk, the A and B chunks (128 rows x 128 B
//                each, fp32, 128-byte swizzle) into a kStages-deep ring
//   warps 4..7   split: rewrite each landed chunk in place as hi() and write lo() into the
//                stage's second half (element by element, so both share the swizzled layout)
//   warp 9       MMA issuer (one thread): per chunk and 8-deep k-step three kind::tf32 MMAs
//                (M = N = 128) into the tile's accumulator (two TMEM buffers of 128 columns)
//   warps 0..3   epilogue: TMEM -> registers (warp w reads lanes 32w..32w+31: one output row
//                per thread), + residual, -> global; overlaps the next tile's main loop
// Every wait is bounded; on a timeout the CTA raises its abort flag, the roles leave their
// loops, in-flight copies and MMAs are drained and the tensor memory is freed.
#pragma once

#include "veda_ptx.cuh"

namespace veda {
namespace sgemm {

constexpr int kThreads = 320;
constexpr int kStages = 3;
constexpr uint32_t kChunkB = 16384;                 // 128 rows x 32 fp32
constexpr uint32_t kOffA = 0, kOffB = kChunkB;      // hi planes (TMA destinations)
constexpr uint32_t kOffLo = 2 * kChunkB;            // lo planes: A at +kOffLo, B at +kOffLo + kChunkB
constexpr uint32_t kStageB = 4 * kChunkB;           // 64 KB
constexpr uint32_t kSmemBytes = kStages * kStageB + 1024;   // + alignment slack
constexpr uint32_t kTmemCols = 256;                 // two 128-column accumulators
constexpr uint32_t kIdesc = idesc_tf32_f32(128, 128);
constexpr int kSplitThreads = 128;
constexpr int kEpiThreads = 128;

enum : int32_t { kModeProject = 0, kModeScores = 1 };

struct Args {
  int32_t mode;
  int32_t nT;          // rows per (b, h) of A and of the output
  int32_t N;           // output columns (128 for the projection, nT for the scores)
  int32_t k_chunks;    // K / 32
  int32_t tiles_m, tiles_n;
  int32_t BH, H;
  int64_t tiles;       // problems * tiles_m * tiles_n
  const float* res[2]; // projection: pooled_q, pooled_k (residual = first 128 of each 384-row)
  float* out;          // projection: qhat/khat [2][BH][nT][128]; scores: [BH][nT][nT]
};

struct Tile {
  int32_t which;       // operand pair (projection: 0 = q, 1 = k)
  int32_t z;           // b * H + h
  int32_t m0, n0;      // first output row / column
  int32_t a_row, b_row;
};

__device__ __forceinline__ Tile tile_of(const Args& a, int64_t t) {
  const int64_t per = static_cast<int64_t>(a.tiles_m) * a.tiles_n;
  const int32_t p = static_cast<int32_t>(t / per);
  const int32_t rem = static_cast<int32_t>(t - static_cast<int64_t>(p) * per);
  Tile r;
  r.m0 = (rem / a.tiles_n) * 128;
  r.n0 = (rem % a.tiles_n) * 128;
  if (a.mode == kModeProject) {
    r.which = p / a.BH;
    r.z = p % a.BH;
    r.a_row = r.z * a.nT + r.m0;
    r.b_row = (r.z % a.H) * 128;          // W[h]: 128 rows of 384
  } else {
    r.which = 0;
    r.z = p;
    r.a_row = r.z * a.nT + r.m0;          // qhat rows
    r.b_row = (a.BH + r.z) * a.nT + r.n0; // khat rows
  }
  return r;
}

struct Bars {
  uint64_t full[kStages];      // TMA landed (tx bytes)
  uint64_t split[kStages];     // hi/lo planes written (kSplitThreads arrivals)
  uint64_t empty[kStages];     // MMAs of the stage done (tcgen05.commit)
  uint64_t acc_full[2];        // tile's accumulator complete (tcgen05.commit)
  uint64_t acc_empty[2];       // epilogue has read the accumulator (kEpiThreads arrivals)
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ void role_producer(const Args& a, Bars& bars, uint32_t sb, const CUtensorMap* mA0,
                                              const CUtensorMap* mA1, const CUtensorMap* mB0,
                                              const CUtensorMap* mB1, volatile int* abort) {
  uint32_t g = 0;   // chunks issued
  for (int64_t t = blockIdx.x; t < a.tiles && !*abort; t += gridDim.x) {
    const Tile tl = tile_of(a, t);
    const CUtensorMap* mA = tl.which ? mA1 : mA0;
    const CUtensorMap* mB = tl.which ? mB1 : mB0;
    for (int32_t c = 0; c < a.k_chunks; ++c, ++g) {
      const uint32_t s = g % kStages;
      if (g >= kStages && !mbar_wait(smem_u32(&bars.empty[s]), (g / kStages - 1) & 1, abort, 60)) {
        t = a.tiles;   // leave both loops
        break;
      }
      const uint32_t st = sb + s * kStageB;
      mbar_arrive_expect_tx(smem_u32(&bars.full[s]), 2 * kChunkB);
      tma_load_2d(st + kOffA, mA, smem_u32(&bars.full[s]), c * 32, tl.a_row);
      tma_load_2d(st + kOffB, mB, smem_u32(&bars.full[s]), c * 32, tl.b_row);
    }
  }
  if (*abort) {   // copies still in flight land before the CTA releases its shared memory
    for (uint32_t i = g > kStages ? g - kStages : 0; i < g; ++i)
      mbar_wait(smem_u32(&bars.full[i % kStages]), (i / kStages) & 1, nullptr, 61);
  }
}

// hi() in place and lo() beside it, for the A and B chunks of one stage (32 KB of fp32).
__device__ __forceinline__ void role_split(const Args& a, Bars& bars, uint8_t* smem, uint32_t tid,
                                           volatile int* abort) {
  uint32_t g = 0;
  for (int64_t t = blockIdx.x; t < a.tiles; t += gridDim.x) {
    for (int32_t c = 0; c < a.k_chunks; ++c, ++g) {
      const uint32_t s = g % kStages;
      if (!mbar_wait(smem_u32(&bars.full[s]), (g / kStages) & 1, abort, 62)) return;
      float4* hi = reinterpret_cast<float4*>(smem + s * kStageB);
      float4* lo = reinterpret_cast<float4*>(smem + s * kStageB + kOffLo);
#pragma unroll 4
      for (uint32_t i = tid; i < 2 * kChunkB / 16; i += kSplitThreads) {
        const float4 x = hi[i];
        float4 h, l;
        h.x = tf32_round(x.x); l.x = tf32_round(x.x - h.x);
        h.y = tf32_round(x.y); l.y = tf32_round(x.y - h.y);
        h.z = tf32_round(x.z); l.z = tf32_round(x.z - h.z);
        h.w = tf32_round(x.w); l.w = tf32_round(x.w - h.w);
        hi[i] = h;
        lo[i] = l;
      }
      fence_proxy_async_smem();   // the tensor core reads these planes through the async proxy
      mbar_arrive(smem_u32(&bars.split[s]));
    }
  }
}

__device__ __forceinline__ void role_mma(const Args& a, Bars& bars, uint32_t sb, uint32_t tmem,
                                         volatile int* abort) {
  uint32_t g = 0, it = 0;
  for (int64_t t = blockIdx.x; t < a.tiles; t += gridDim.x, ++it) {
    const uint32_t ab = it & 1;
    if (it >= 2 && !mbar_wait(smem_u32(&bars.acc_empty[ab]), ((it >> 1) - 1) & 1, abort, 63)) break;
    tc_fence_after();
    const uint32_t d = tmem + ab * 128;
    bool ok = true;
    for (int32_t c = 0; c < a.k_chunks; ++c, ++g) {
      const uint32_t s = g % kStages;
      if (!mbar_wait(smem_u32(&bars.split[s]), (g / kStages) & 1, abort, 64)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t st = sb + s * kStageB;
      const uint64_t dA = smem_desc_sw128(st + kOffA, 16, 1024);
      const uint64_t dB = smem_desc_sw128(st + kOffB, 16, 1024);
      const uint64_t dAl = smem_desc_sw128(st + kOffLo + kOffA, 16, 1024);
      const uint64_t dBl = smem_desc_sw128(st + kOffLo + kOffB, 16, 1024);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {   // 8 tf32 = 32 bytes per k-step: +2 in 16-byte units
        const uint64_t o = static_cast<uint64_t>(kk * 2);
        mma_ss_tf32(d, dAl + o, dB + o, kIdesc, (c > 0 || kk > 0) ? 1u : 0u);
        mma_ss_tf32(d, dA + o, dBl + o, kIdesc, 1u);
        mma_ss_tf32(d, dA + o, dB + o, kIdesc, 1u);
      }
      tc_commit(smem_u32(&bars.empty[s]));
    }
    if (!ok) break;
    tc_commit(smem_u32(&bars.acc_full[ab]));
  }
  tc_commit(smem_u32(&bars.drain));
  mbar_wait(smem_u32(&bars.drain), 0, nullptr, 65);
}

__device__ __forceinline__ void role_epilogue(const Args& a, Bars& bars, uint32_t tmem, uint32_t warp,
                                              uint32_t lane, volatile int* abort) {
  uint32_t it = 0;
  const bool vec = (a.N % 4) == 0;
  for (int64_t t = blockIdx.x; t < a.tiles; t += gridDim.x, ++it) {
    const Tile tl = tile_of(a, t);
    const uint32_t ab = it & 1;
    if (!mbar_wait(smem_u32(&bars.acc_full[ab]), (it >> 1) & 1, abort, 66)) return;
    tc_fence_after();
    const int32_t m = tl.m0 + static_cast<int32_t>(warp * 32 + lane);   // this thread's output row
    const bool row_ok = m < a.nT;
    float* orow;
    const float* rrow = nullptr;
    if (a.mode == kModeProject) {
      orow = a.out + (static_cast<int64_t>(tl.which) * a.BH + tl.z) * a.nT * 128 + static_cast<int64_t>(m) * 128;
      rrow = a.res[tl.which] + (static_cast<int64_t>(tl.z) * a.nT + m) * 384;
    } else {
      orow = a.out + static_cast<int64_t>(tl.z) * a.nT * a.nT + static_cast<int64_t>(m) * a.nT;
    }
    const uint32_t taddr = tmem + ((warp * 32) << 16) + ab * 128;
#pragma unroll 1
    for (int cc = 0; cc < 4; ++cc) {
      uint32_t r[32];
      tmem_ld32_sync(taddr + cc * 32, r);
      const int32_t n0 = tl.n0 + cc * 32;
      if (!row_ok || n0 >= a.N) continue;
      if (vec && n0 + 32 <= a.N) {
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          float4 v = make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]), __uint_as_float(r[j + 2]),
                                 __uint_as_float(r[j + 3]));
          if (rrow) {
            const float4 x = *reinterpret_cast<const float4*>(rrow + n0 + j);
            v.x += x.x; v.y += x.y; v.z += x.z; v.w += x.w;
          }
          *reinterpret_cast<float4*>(orow + n0 + j) = v;
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          if (n0 + j < a.N) {
            float v = __uint_as_float(r[j]);
            if (rrow) v += rrow[n0 + j];
            orow[n0 + j] = v;
          }
        }
      }
    }
    tc_fence_before();
    mbar_arrive(smem_u32(&bars.acc_empty[ab]));
  }
}

__global__ void __launch_bounds__(kThreads, 1)
nt_gemm_3xtf32_kernel(const __grid_constant__ CUtensorMap mA0, const __grid_constant__ CUtensorMap mA1,
                      const __grid_constant__ CUtensorMap mB0, const __grid_constant__ CUtensorMap mB1,
                      const Args a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ Bars bars;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const uint32_t tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  volatile int* abort = &bars.abort;

  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(smem_u32(&bars.full[i]), 1);
      mbar_init(smem_u32(&bars.split[i]), kSplitThreads);
      mbar_init(smem_u32(&bars.empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bars.acc_full[i]), 1);
      mbar_init(smem_u32(&bars.acc_empty[i]), kEpiThreads);
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
    prefetch_tensormap(&mA0);
    prefetch_tensormap(&mA1);
    prefetch_tensormap(&mB0);
    prefetch_tensormap(&mB1);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;

  if (warp < 4)
    role_epilogue(a, bars, tmem, warp, lane, abort);
  else if (warp < 8)
    role_split(a, bars, smem, tid - 128, abort);
  else if (warp == 8 && lane == 0)
    role_producer(a, bars, sb, &mA0, &mA1, &mB0, &mB1, abort);
  else if (warp == 9 && lane == 0)
    role_mma(a, bars, sb, tmem, abort);

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace sgemm
}  // namespace veda
