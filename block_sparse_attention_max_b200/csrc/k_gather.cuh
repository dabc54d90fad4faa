// k_gather.cuh -- steps 1, 2 and 6: tile gather (permute), tile pooling, scatter back.
//
// All three stream HBM and move 256-byte token rows (128 bf16 of one head). The gather
// side of the permute and the scatter side of the unpermute address every row on its
// own, so they are written as wide coalesced register copies: 16 threads move one row
// with 16-byte accesses, a warp moves two rows per instruction, and every thread keeps
// eight 16-byte loads in flight before its first store (memory-level parallelism
// without a per-row copy request). The tile side of each copy is one contiguous 32 KB
// block. Pooling reads each tile once: one warp reduces a whole tile with 16-byte loads
// and no shared memory or block barrier.
#pragma once

#include "veda_ptx.cuh"

namespace veda {

constexpr uint32_t kRowBytes = 256;                 // one token of one head: 128 bf16
constexpr uint32_t kTileBytes = 128 * kRowBytes;    // one tile: 32 KB
constexpr int kCopyThreads = 256;                   // 16 row-groups x 16 chunks per tile pass

struct GatherArgs {
  const uint8_t* src;
  uint8_t* dst;
  const int32_t* map;    // [H][Npad]
  int32_t B, N, H, Npad, nT;
  int64_t units;         // B * H * nT
};

// Units in head-minor order (b, t, h): the CTAs running at one time take the same tile of
// many heads, so together they read (permute) or write (unpermute) whole raster token rows
// of H * 256 bytes instead of one head's 256 bytes out of each.
__device__ __forceinline__ void unit_coords(int64_t u, int32_t H, int32_t nT, int32_t& b,
                                            int32_t& h, int32_t& t) {
  h = static_cast<int32_t>(u % H);
  const int64_t bt = u / H;
  t = static_cast<int32_t>(bt % nT);
  b = static_cast<int32_t>(bt / nT);
}

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ void st_v4(void* p, uint4 v) {
  asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

// ------------------------------------------------------------------------------------
// Step 1: x[B][N][H][128] -> x_tiled[B][H][Npad][128], pad slots zero.
// Thread t of a CTA handles 16-byte chunk (t & 15) of rows (t >> 4) + 16 i, i < 8.
// ------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kCopyThreads) permute_kernel(const GatherArgs a) {
  const uint32_t c = threadIdx.x & 15, r0 = threadIdx.x >> 4;
  for (int64_t u = blockIdx.x; u < a.units; u += gridDim.x) {
    int32_t b, h, t;
    unit_coords(u, a.H, a.nT, b, h, t);
    const int32_t* m = a.map + static_cast<int64_t>(h) * a.Npad + static_cast<int64_t>(t) * 128;
    int32_t tok[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) tok[i] = __ldg(m + r0 + 16 * i);
    uint4 v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[i] = make_uint4(0, 0, 0, 0);
      if (tok[i] >= a.N) flag_status(ST_BAD_MAP);
      if (tok[i] >= 0 && tok[i] < a.N)
        v[i] = ld_stream(a.src + ((static_cast<int64_t>(b) * a.N + tok[i]) * a.H + h) * kRowBytes + c * 16);
    }
    uint8_t* dst = a.dst + ((static_cast<int64_t>(b) * a.H + h) * a.Npad + static_cast<int64_t>(t) * 128) * kRowBytes;
#pragma unroll
    for (int i = 0; i < 8; ++i) st_v4(dst + (r0 + 16 * i) * kRowBytes + c * 16, v[i]);
  }
}

// ------------------------------------------------------------------------------------
// Step 6: o_tiled[B][H][Npad][128] -> o[B][N][H][128] for slots that map to a token.
// ------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kCopyThreads) unpermute_kernel(const GatherArgs a) {
  const uint32_t c = threadIdx.x & 15, r0 = threadIdx.x >> 4;
  for (int64_t u = blockIdx.x; u < a.units; u += gridDim.x) {
    int32_t b, h, t;
    unit_coords(u, a.H, a.nT, b, h, t);
    const int32_t* m = a.map + static_cast<int64_t>(h) * a.Npad + static_cast<int64_t>(t) * 128;
    const uint8_t* src = a.src + ((static_cast<int64_t>(b) * a.H + h) * a.Npad + static_cast<int64_t>(t) * 128) * kRowBytes;
    int32_t tok[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) tok[i] = __ldg(m + r0 + 16 * i);
    uint4 v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (tok[i] >= 0 && tok[i] < a.N) v[i] = ld_stream(src + (r0 + 16 * i) * kRowBytes + c * 16);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (tok[i] >= a.N) flag_status(ST_BAD_MAP);
      if (tok[i] >= 0 && tok[i] < a.N)
        st_v4(a.dst + ((static_cast<int64_t>(b) * a.N + tok[i]) * a.H + h) * kRowBytes + c * 16, v[i]);
    }
  }
}

// ------------------------------------------------------------------------------------
// Step 2: pooled[B][H][nT][3][128] = mean / max / min over each tile's valid prefix.
// One warp per tile: lane l reduces chunk (l & 15) = channels 8(l&15)..+7 over rows
// (l >> 4) + 2 i; the two halves of the warp are combined with one shuffle.
// ------------------------------------------------------------------------------------
constexpr int kPoolThreads = 256;

struct PoolArgs {
  const uint8_t* x;       // [B][H][nT*128][128] bf16
  const int32_t* valid;   // [H][nT]
  float* out;             // [B][H][nT][3][128]
  int32_t B, H, nT;
  int64_t units;
};

__global__ void __launch_bounds__(kPoolThreads) pool_kernel(const PoolArgs a) {
  const uint32_t lane = threadIdx.x & 31;
  const uint32_t c = lane & 15, half = lane >> 4;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (kPoolThreads / 32);
  for (int64_t u = static_cast<int64_t>(blockIdx.x) * (kPoolThreads / 32) + (threadIdx.x >> 5); u < a.units;
       u += warps) {
    int32_t b, h, t;
    unit_coords(u, a.H, a.nT, b, h, t);
    const int64_t lin = (static_cast<int64_t>(b) * a.H + h) * a.nT + t;   // tile index in memory
    int32_t nv = a.valid[static_cast<int64_t>(h) * a.nT + t];
    nv = nv < 0 ? 0 : (nv > 128 ? 128 : nv);
    const uint8_t* tile = a.x + lin * kTileBytes + c * 16;
    float sum[8];
    __nv_bfloat162 mx[4], mn[4];
#pragma unroll
    for (int k = 0; k < 8; ++k) sum[k] = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      mx[k] = __floats2bfloat162_rn(-INFINITY, -INFINITY);
      mn[k] = __floats2bfloat162_rn(INFINITY, INFINITY);
    }
    for (int32_t r0 = 0; r0 < nv; r0 += 16) {
      uint4 v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int32_t r = r0 + static_cast<int32_t>(half) + 2 * i;
        if (r < nv) v[i] = ld_stream(tile + r * kRowBytes);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int32_t r = r0 + static_cast<int32_t>(half) + 2 * i;
        if (r < nv) {
          const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v[i]);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float2 f = __bfloat1622float2(p[k]);
            sum[2 * k] += f.x;
            sum[2 * k + 1] += f.y;
            mx[k] = __hmax2(mx[k], p[k]);
            mn[k] = __hmin2(mn[k], p[k]);
          }
        }
      }
    }
    float fmx[8], fmn[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 a2 = __bfloat1622float2(mx[k]), b2 = __bfloat1622float2(mn[k]);
      fmx[2 * k] = a2.x; fmx[2 * k + 1] = a2.y;
      fmn[2 * k] = b2.x; fmn[2 * k + 1] = b2.y;
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      sum[k] += __shfl_xor_sync(0xffffffffu, sum[k], 16);
      fmx[k] = fmaxf(fmx[k], __shfl_xor_sync(0xffffffffu, fmx[k], 16));
      fmn[k] = fminf(fmn[k], __shfl_xor_sync(0xffffffffu, fmn[k], 16));
    }
    if (half == 0) {
      float4* o = reinterpret_cast<float4*>(a.out + lin * 384 + c * 8);
      if (nv > 0) {
        const float inv = 1.0f / static_cast<float>(nv);
        o[0] = make_float4(sum[0] * inv, sum[1] * inv, sum[2] * inv, sum[3] * inv);
        o[1] = make_float4(sum[4] * inv, sum[5] * inv, sum[6] * inv, sum[7] * inv);
        o[32] = make_float4(fmx[0], fmx[1], fmx[2], fmx[3]);
        o[33] = make_float4(fmx[4], fmx[5], fmx[6], fmx[7]);
        o[64] = make_float4(fmn[0], fmn[1], fmn[2], fmn[3]);
        o[65] = make_float4(fmn[4], fmn[5], fmn[6], fmn[7]);
      } else {
        const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
        o[0] = z; o[1] = z; o[32] = z; o[33] = z; o[64] = z; o[65] = z;
      }
    }
  }
}

// ------------------------------------------------------------------------------------
// Steps 1 + 2 fused (a variant; the two calls also stay separate): gather a tile as
// permute_kernel does and reduce mean / max / min over its valid slots on the way, so the
// tiled tensor is not read a second time. One warp per tile, as in pool_kernel: lane l
// moves 16-byte chunk (l & 15) of rows (l >> 4) + 2 i, 16 rows per pass, and keeps the
// running sums / maxima / minima of its eight channels in registers; one shuffle combines
// the two row groups at the end. No shared memory and no block barrier, so the warps of a
// CTA never wait for one another and the gather stream does not stall between tiles.
// ------------------------------------------------------------------------------------
struct PermPoolArgs {
  GatherArgs g;
  const int32_t* valid;   // [H][nT]
  float* pooled;          // [B][H][nT][3][128]
};

__global__ void __launch_bounds__(kPoolThreads) permute_pool_kernel(const PermPoolArgs p) {
  const GatherArgs& a = p.g;
  const uint32_t lane = threadIdx.x & 31;
  const uint32_t c = lane & 15, half = lane >> 4;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (kPoolThreads / 32);
  for (int64_t u = static_cast<int64_t>(blockIdx.x) * (kPoolThreads / 32) + (threadIdx.x >> 5); u < a.units;
       u += warps) {
    int32_t b, h, t;
    unit_coords(u, a.H, a.nT, b, h, t);
    const int64_t lin = (static_cast<int64_t>(b) * a.H + h) * a.nT + t;   // tile index in memory
    int32_t nv = p.valid[static_cast<int64_t>(h) * a.nT + t];
    nv = nv < 0 ? 0 : (nv > 128 ? 128 : nv);
    const int32_t* m = a.map + static_cast<int64_t>(h) * a.Npad + static_cast<int64_t>(t) * 128 + half;
    const uint8_t* src = a.src + (static_cast<int64_t>(b) * a.N * a.H + h) * kRowBytes + c * 16;
    const int64_t tok_stride = static_cast<int64_t>(a.H) * kRowBytes;
    uint8_t* dst = a.dst + lin * kTileBytes + half * kRowBytes + c * 16;
    float sum[8], mx[8], mn[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) { sum[k] = 0.f; mx[k] = -INFINITY; mn[k] = INFINITY; }
#pragma unroll 1
    for (int32_t r0 = 0; r0 < 128; r0 += 16) {
      int32_t tok[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) tok[i] = __ldg(m + r0 + 2 * i);
      uint4 v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        v[i] = make_uint4(0, 0, 0, 0);
        if (tok[i] >= a.N) flag_status(ST_BAD_MAP);
        if (tok[i] >= 0 && tok[i] < a.N) v[i] = ld_stream(src + tok[i] * tok_stride);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) st_v4(dst + (r0 + 2 * i) * kRowBytes, v[i]);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (r0 + static_cast<int32_t>(half) + 2 * i < nv) {
          const __nv_bfloat162* q = reinterpret_cast<const __nv_bfloat162*>(&v[i]);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float2 f = __bfloat1622float2(q[k]);
            sum[2 * k] += f.x;
            sum[2 * k + 1] += f.y;
            mx[2 * k] = fmaxf(mx[2 * k], f.x);
            mx[2 * k + 1] = fmaxf(mx[2 * k + 1], f.y);
            mn[2 * k] = fminf(mn[2 * k], f.x);
            mn[2 * k + 1] = fminf(mn[2 * k + 1], f.y);
          }
        }
      }
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      sum[k] += __shfl_xor_sync(0xffffffffu, sum[k], 16);
      mx[k] = fmaxf(mx[k], __shfl_xor_sync(0xffffffffu, mx[k], 16));
      mn[k] = fminf(mn[k], __shfl_xor_sync(0xffffffffu, mn[k], 16));
    }
    if (half == 0) {
      float4* o = reinterpret_cast<float4*>(p.pooled + lin * 384 + c * 8);
      if (nv > 0) {
        const float inv = 1.0f / static_cast<float>(nv);
        o[0] = make_float4(sum[0] * inv, sum[1] * inv, sum[2] * inv, sum[3] * inv);
        o[1] = make_float4(sum[4] * inv, sum[5] * inv, sum[6] * inv, sum[7] * inv);
        o[32] = make_float4(mx[0], mx[1], mx[2], mx[3]);
        o[33] = make_float4(mx[4], mx[5], mx[6], mx[7]);
        o[64] = make_float4(mn[0], mn[1], mn[2], mn[3]);
        o[65] = make_float4(mn[4], mn[5], mn[6], mn[7]);
      } else {
        const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
        o[0] = z; o[1] = z; o[32] = z; o[33] = z; o[64] = z; o[65] = z;
      }
    }
  }
}

}  // namespace veda
