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
// operand (the "3xTF32" scheme): x = hi(x) + lo(x) with hi(x) = x with its 13 low mantissa
// bits cleared (exactly a tf32 value) and lo(x) = x - hi(x) (exact in fp32; the tensor core
// reads it to tf32 precision), and
//   A B^T ~= hi(A) hi(B)^T + hi(A) lo(B)^T + lo(A) hi(B)^T,
// whose dropped term lo(A) lo(B)^T and the tf32 precision of lo are ~2^-20 of |A||B| -- far
// below the tolerance -- while every product runs at the tensor-core tf32 rate with an
// fp32 accumulator in tensor memory. The split is one logical AND and one subtraction per
// element (no conversion instruction).
//
// Kernel: persistent, one CTA per SM, one 128 x 128 output tile at a time.
//   warp 12      TMA producer: per 32-deep K chunk, the A and B chunks (128 rows x 128 B
//                each, fp32, 128-byte swizzle) into a kStages-deep ring
//   warps 4..11  split: rewrite each landed chunk in place as hi() and write lo() into the
//                stage's second half (element by element, so both share the swizzled layout)
//   warp 13      MMA issuer (one thread): per chunk and 8-deep k-step three kind::tf32 MMAs
//                (M = N = 128) into the tile's accumulator (two TMEM buffers of 128 columns)
//   warps 0..3   epilogue: TMEM -> registers (warp w reads lanes 32w..32w+31: one output row
//                per thread) -> global; overlaps the next tile's main loop
// The projection's residual (the mean, columns 0..127 of the pooled row, i.e. A chunks 0..3)
// is added by the tensor core too: hi(A) I + lo(A) I against a 32 x 32 identity held in shared
// memory, into accumulator columns c*32 .. c*32 + 31, so the epilogue has no global loads.
// Every wait is bounded; on a timeout the CTA raises its abort flag, the roles leave their
// loops, in-flight copies and MMAs are drained and the tensor memory is freed.
#pragma once

#include "k_attn.cuh"   // attn::warp_wait_abort
#include "veda_ptx.cuh"

namespace veda {
namespace sgemm {

constexpr int kThreads = 448;
constexpr int kStages = 3;
constexpr uint32_t kChunkB = 16384;                 // 128 rows x 32 fp32
constexpr uint32_t kOffA = 0, kOffB = kChunkB;      // hi planes (TMA destinations)
constexpr uint32_t kOffLo = 2 * kChunkB;            // lo planes: A at +kOffLo, B at +kOffLo + kChunkB
constexpr uint32_t kStageB = 4 * kChunkB;           // 64 KB
constexpr uint32_t kOffI = kStages * kStageB;       // 32 x 32 identity (tf32, K-major, swizzled)
constexpr uint32_t kSmemBytes = kOffI + 4096 + 1024;   // + alignment slack
constexpr uint32_t kTmemCols = 256;                 // two 128-column accumulators
constexpr uint32_t kIdesc = idesc_tf32_f32(128, 128);
constexpr uint32_t kIdescI = idesc_tf32_f32(128, 32);  // mean chunk x identity: the residual
constexpr int kSplitThreads = 256;
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
  uint64_t split[kStages];     // hi/lo planes written (one arrival per split warp)
  uint64_t empty[kStages];     // MMAs of the stage done (tcgen05.commit)
  uint64_t acc_full[2];        // tile's accumulator complete (tcgen05.commit)
  uint64_t acc_empty[2];       // epilogue has read the accumulator (one arrival per epilogue warp)
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
  // every copy lands before the CTA releases its shared memory, also when another role gave
  // up after this loop ended (in the normal run these phases have long completed)
  for (uint32_t i = g > kStages ? g - kStages : 0; i < g; ++i)
    mbar_wait(smem_u32(&bars.full[i % kStages]), (i / kStages) & 1, nullptr, 61);
}

// x with its 13 low mantissa bits cleared: a tf32 value, and x - tf32_hi(x) is exact.
__device__ __forceinline__ float tf32_hi(float x) { return __uint_as_float(__float_as_uint(x) & 0xFFFFE000u); }

// The 32 x 32 identity in the MMA's K-major, 128-byte-swizzled layout: row n (128 bytes)
// holds 1.0 at k = n; the 16-byte group of element k sits at (k / 4) ^ (n % 8).
__device__ __forceinline__ void build_identity(uint8_t* smem, uint32_t tid) {
  for (uint32_t e = tid; e < 32 * 32; e += kSplitThreads) {
    const uint32_t n = e / 32, k = e % 32;
    *reinterpret_cast<float*>(smem + kOffI + n * 128 + (((k / 4) ^ (n % 8)) * 16) + (k % 4) * 4) =
        n == k ? 1.0f : 0.0f;
  }
  fence_proxy_async_smem();
}

// hi() in place and lo() beside it, for the A and B chunks of one stage (32 KB of fp32).
__device__ __forceinline__ void role_split(const Args& a, Bars& bars, uint8_t* smem, uint32_t tid,
                                           volatile int* abort) {
  uint32_t g = 0;
  for (int64_t t = blockIdx.x; t < a.tiles; t += gridDim.x) {
    for (int32_t c = 0; c < a.k_chunks; ++c, ++g) {
      const uint32_t s = g % kStages;
      if (!attn::warp_wait_abort(smem_u32(&bars.full[s]), (g / kStages) & 1, abort, 62)) return;
      float4* hi = reinterpret_cast<float4*>(smem + s * kStageB);
      float4* lo = reinterpret_cast<float4*>(smem + s * kStageB + kOffLo);
#pragma unroll 4
      for (uint32_t i = tid; i < 2 * kChunkB / 16; i += kSplitThreads) {
        const float4 x = hi[i];
        float4 h, l;
        h.x = tf32_hi(x.x); l.x = x.x - h.x;
        h.y = tf32_hi(x.y); l.y = x.y - h.y;
        h.z = tf32_hi(x.z); l.z = x.z - h.z;
        h.w = tf32_hi(x.w); l.w = x.w - h.w;
        hi[i] = h;
        lo[i] = l;
      }
      fence_proxy_async_smem();   // the tensor core reads these planes through the async proxy
      __syncwarp();
      if ((tid & 31) == 0) mbar_arrive(smem_u32(&bars.split[s]));
    }
  }
}

__device__ __forceinline__ void role_mma(const Args& a, Bars& bars, uint32_t sb, uint32_t tmem,
                                         volatile int* abort) {
  const uint64_t dI = smem_desc_sw128(sb + kOffI, 16, 1024);
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
      // projection: chunks 0..3 of A are the mean, whose columns c*32.. also get the mean
      // itself (the residual): hi(A) I + lo(A) I into accumulator columns c*32 .. c*32 + 31
      const bool residual = a.mode == kModeProject && c < 4;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {   // 8 tf32 = 32 bytes per k-step: +2 in 16-byte units
        const uint64_t o = static_cast<uint64_t>(kk * 2);
        mma_ss_tf32(d, dAl + o, dB + o, kIdesc, (c > 0 || kk > 0) ? 1u : 0u);
        mma_ss_tf32(d, dA + o, dBl + o, kIdesc, 1u);
        mma_ss_tf32(d, dA + o, dB + o, kIdesc, 1u);
        if (residual) {
          mma_ss_tf32(d + c * 32, dAl + o, dI + o, kIdescI, 1u);
          mma_ss_tf32(d + c * 32, dA + o, dI + o, kIdescI, 1u);
        }
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
    if (!attn::warp_wait_abort(smem_u32(&bars.acc_full[ab]), (it >> 1) & 1, abort, 66)) return;
    tc_fence_after();
    const int32_t m = tl.m0 + static_cast<int32_t>(warp * 32 + lane);   // this thread's output row
    const bool row_ok = m < a.nT;
    float* orow;
    if (a.mode == kModeProject) {
      orow = a.out + (static_cast<int64_t>(tl.which) * a.BH + tl.z) * a.nT * 128 + static_cast<int64_t>(m) * 128;
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
        for (int j = 0; j < 32; j += 4)
          *reinterpret_cast<float4*>(orow + n0 + j) =
              make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]), __uint_as_float(r[j + 2]),
                          __uint_as_float(r[j + 3]));
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (n0 + j < a.N) orow[n0 + j] = __uint_as_float(r[j]);
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&bars.acc_empty[ab]));
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
      mbar_init(smem_u32(&bars.split[i]), kSplitThreads / 32);
      mbar_init(smem_u32(&bars.empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bars.acc_full[i]), 1);
      mbar_init(smem_u32(&bars.acc_empty[i]), kEpiThreads / 32);
    }
    mbar_init(smem_u32(&bars.drain), 1);
    bars.abort = 0;
    fence_mbar_init();
  }
  if (warp == 13) {
    tmem_alloc(smem_u32(&bars.tmem_base), kTmemCols);
    tmem_relinquish();
  }
  if (warp >= 4 && warp < 12) build_identity(smem, tid - 128);
  if (warp == 12 && lane == 0) {
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
  else if (warp < 12)
    role_split(a, bars, smem, tid - 128, abort);
  else if (warp == 12 && lane == 0)
    role_producer(a, bars, sb, &mA0, &mA1, &mB0, &mB1, abort);
  else if (warp == 13 && lane == 0)
    role_mma(a, bars, sb, tmem, abort);

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 13) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace sgemm
}  // namespace veda
