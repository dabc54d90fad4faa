// k_gather.cuh -- steps 1, 2 and 6: tile gather (permute), tile pooling, scatter back.
//
// All three stream HBM. A CTA walks a strided range of (batch, head, tile) units and
// keeps a ring of 32 KB tile buffers in shared memory filled by bulk asynchronous
// copies (the TMA engine): per-row 256-byte copies for the gather side of the
// permute, one contiguous copy per tile elsewhere. Completion is tracked by one
// mbarrier per ring slot (transaction bytes); writes go out as bulk stores.
#pragma once

#include "veda_ptx.cuh"

namespace veda {

constexpr uint32_t kRowBytes = 256;                 // one token of one head: 128 bf16
constexpr uint32_t kTileBytes = 128 * kRowBytes;    // one tile: 32 KB

struct GatherArgs {
  const uint8_t* src;
  uint8_t* dst;
  const int32_t* map;    // [H][Npad]
  int32_t B, N, H, Npad, nT;
  int64_t units;         // B * H * nT
};

__device__ __forceinline__ void unit_coords(int64_t u, int32_t H, int32_t nT, int32_t& b,
                                            int32_t& h, int32_t& t) {
  t = static_cast<int32_t>(u % nT);
  const int64_t bh = u / nT;
  h = static_cast<int32_t>(bh % H);
  b = static_cast<int32_t>(bh / H);
}

// Lane 0 waits (bounded) for the phase; the verdict is broadcast so that the whole
// warp takes the same path, and every lane then observes the completed phase itself
// (acquire of the bulk-copied data).
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, uint32_t site) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, nullptr, site);
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (ok) ok = mbar_try_wait(bar, parity);
  return __all_sync(0xffffffffu, ok);
}

// ------------------------------------------------------------------------------------
// Step 1: x[B][N][H][128] -> x_tiled[B][H][Npad][128]. One warp per CTA.
// ------------------------------------------------------------------------------------
constexpr int kPermStages = 6;

__global__ void __launch_bounds__(32, 1) permute_kernel(const GatherArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[kPermStages];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t lane = threadIdx.x;
  const uint32_t sbase = smem_u32(smem);
  if (lane == 0) {
    for (int s = 0; s < kPermStages; ++s) mbar_init(smem_u32(&full_bar[s]), 1);
    fence_mbar_init();
  }
  __syncwarp();

  const int64_t first = blockIdx.x, stride = gridDim.x;
  const int64_t n_local = first < a.units ? (a.units - first + stride - 1) / stride : 0;

  auto issue = [&](int64_t k) {
    const int s = static_cast<int>(k % kPermStages);
    int32_t b, h, t;
    unit_coords(first + k * stride, a.H, a.nT, b, h, t);
    const int32_t* m = a.map + static_cast<int64_t>(h) * a.Npad + static_cast<int64_t>(t) * 128;
    int32_t tok[4];
    uint32_t nrows = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      tok[i] = m[lane + 32 * i];
      if (tok[i] >= a.N) {
        flag_status(ST_BAD_MAP);
        tok[i] = -1;
      }
      nrows += tok[i] >= 0;
    }
    nrows = __reduce_add_sync(0xffffffffu, nrows);
    const uint32_t bar = smem_u32(&full_bar[s]);
    if (lane == 0) mbar_arrive_expect_tx(bar, nrows * kRowBytes);
    __syncwarp();
    const uint32_t buf = sbase + s * kTileBytes;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t r = lane + 32 * i;
      if (tok[i] >= 0) {
        const uint8_t* src =
            a.src + ((static_cast<int64_t>(b) * a.N + tok[i]) * a.H + h) * static_cast<int64_t>(kRowBytes);
        bulk_g2s(buf + r * kRowBytes, src, kRowBytes, bar);
      } else {
        uint4* z = reinterpret_cast<uint4*>(smem + s * kTileBytes + r * kRowBytes);
#pragma unroll
        for (int c = 0; c < 16; ++c) z[c] = make_uint4(0, 0, 0, 0);
      }
    }
    fence_proxy_async_smem();   // zero rows written by this lane -> visible to the bulk store
  };

  const int64_t pro = n_local < kPermStages ? n_local : kPermStages;
  for (int64_t k = 0; k < pro; ++k) issue(k);

  int64_t k = 0;
  for (; k < n_local; ++k) {
    const int s = static_cast<int>(k % kPermStages);
    if (!warp_wait(smem_u32(&full_bar[s]), static_cast<uint32_t>((k / kPermStages) & 1), 1)) break;
    __syncwarp();
    if (lane == 0) {
      int32_t b, h, t;
      unit_coords(first + k * stride, a.H, a.nT, b, h, t);
      uint8_t* dst = a.dst + ((static_cast<int64_t>(b) * a.H + h) * a.Npad + static_cast<int64_t>(t) * 128) *
                                 static_cast<int64_t>(kRowBytes);
      bulk_s2g(dst, sbase + s * kTileBytes, kTileBytes);
      bulk_commit();
      bulk_wait_read<1>();      // the store issued one iteration ago has read its buffer
    }
    __syncwarp();
    if (k >= 1 && k - 1 + kPermStages < n_local) issue(k - 1 + kPermStages);
  }
  if (k < n_local) {
    // a wait ran out: let every copy still in flight land before the CTA exits
    for (int64_t j = k; j < n_local && j < k + kPermStages; ++j)
      warp_wait(smem_u32(&full_bar[j % kPermStages]), static_cast<uint32_t>((j / kPermStages) & 1), 2);
  }
  if (lane == 0) bulk_wait<0>();
  __syncwarp();
}

// ------------------------------------------------------------------------------------
// Step 6: o_tiled[B][H][Npad][128] -> o[B][N][H][128] (valid slots only). One warp per CTA.
// ------------------------------------------------------------------------------------
constexpr int kUnpermStages = 6;

__global__ void __launch_bounds__(32, 1) unpermute_kernel(const GatherArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[kUnpermStages];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t lane = threadIdx.x;
  const uint32_t sbase = smem_u32(smem);
  if (lane == 0) {
    for (int s = 0; s < kUnpermStages; ++s) mbar_init(smem_u32(&full_bar[s]), 1);
    fence_mbar_init();
  }
  __syncwarp();

  const int64_t first = blockIdx.x, stride = gridDim.x;
  const int64_t n_local = first < a.units ? (a.units - first + stride - 1) / stride : 0;

  auto map_of = [&](int64_t k, int32_t& b, int32_t& h, int32_t& t) {
    unit_coords(first + k * stride, a.H, a.nT, b, h, t);
    return a.map + static_cast<int64_t>(h) * a.Npad + static_cast<int64_t>(t) * 128;
  };
  auto issue = [&](int64_t k) {
    const int s = static_cast<int>(k % kUnpermStages);
    int32_t b, h, t;
    const int32_t* m = map_of(k, b, h, t);
    int32_t last = -1;   // highest slot that maps to a token: only [0, last] is loaded
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int32_t tok = m[lane + 32 * i];
      if (tok >= 0 && tok < a.N) last = static_cast<int32_t>(lane + 32 * i);
    }
    last = __reduce_max_sync(0xffffffffu, last);
    if (lane == 0) {
      const uint32_t bar = smem_u32(&full_bar[s]);
      const uint32_t bytes = static_cast<uint32_t>(last + 1) * kRowBytes;
      mbar_arrive_expect_tx(bar, bytes);
      if (bytes) {
        const uint8_t* src = a.src + ((static_cast<int64_t>(b) * a.H + h) * a.Npad +
                                      static_cast<int64_t>(t) * 128) * static_cast<int64_t>(kRowBytes);
        bulk_g2s(sbase + s * kTileBytes, src, bytes, bar);
      }
    }
  };

  const int64_t pro = n_local < kUnpermStages ? n_local : kUnpermStages;
  for (int64_t k = 0; k < pro; ++k) issue(k);

  int64_t k = 0;
  for (; k < n_local; ++k) {
    const int s = static_cast<int>(k % kUnpermStages);
    if (!warp_wait(smem_u32(&full_bar[s]), static_cast<uint32_t>((k / kUnpermStages) & 1), 3)) break;
    int32_t b, h, t;
    const int32_t* m = map_of(k, b, h, t);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t r = lane + 32 * i;
      const int32_t tok = m[r];
      if (tok >= a.N) flag_status(ST_BAD_MAP);
      if (tok >= 0 && tok < a.N) {
        uint8_t* dst = a.dst + ((static_cast<int64_t>(b) * a.N + tok) * a.H + h) * static_cast<int64_t>(kRowBytes);
        bulk_s2g(dst, sbase + s * kTileBytes + r * kRowBytes, kRowBytes);
      }
    }
    bulk_commit();
    bulk_wait_read<1>();   // this lane's stores of the previous iteration have read their rows
    __syncwarp();
    if (k >= 1 && k - 1 + kUnpermStages < n_local) issue(k - 1 + kUnpermStages);
  }
  if (k < n_local) {
    for (int64_t j = k; j < n_local && j < k + kUnpermStages; ++j)
      warp_wait(smem_u32(&full_bar[j % kUnpermStages]), static_cast<uint32_t>((j / kUnpermStages) & 1), 4);
  }
  bulk_wait<0>();
  __syncwarp();
}

// ------------------------------------------------------------------------------------
// Step 2: pooled[B][H][nT][3][128] = mean / max / min over each tile's valid prefix.
// 256 threads: thread t reduces 16-byte chunk (t & 15) over rows (t >> 4) + 16 i.
// ------------------------------------------------------------------------------------
constexpr int kPoolStages = 5;
constexpr int kPoolThreads = 256;

struct PoolArgs {
  const uint8_t* x;       // [B][H][nT*128][128] bf16
  const int32_t* valid;   // [H][nT]
  float* out;             // [B][H][nT][3][128]
  int32_t B, H, nT;
  int64_t units;
};

__global__ void __launch_bounds__(kPoolThreads, 1) pool_kernel(const PoolArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[kPoolStages];
  __shared__ float red[8][3][128];          // per-warp partials
  __shared__ int32_t nvalid_s[kPoolStages];
  __shared__ int32_t ok_s;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t tid = threadIdx.x;
  const uint32_t sbase = smem_u32(smem);
  if (tid == 0) {
    for (int s = 0; s < kPoolStages; ++s) mbar_init(smem_u32(&full_bar[s]), 1);
    fence_mbar_init();
  }
  __syncthreads();

  const int64_t first = blockIdx.x, stride = gridDim.x;
  const int64_t n_local = first < a.units ? (a.units - first + stride - 1) / stride : 0;

  auto issue = [&](int64_t k) {    // thread 0 only
    const int s = static_cast<int>(k % kPoolStages);
    int32_t b, h, t;
    unit_coords(first + k * stride, a.H, a.nT, b, h, t);
    int32_t nv = a.valid[static_cast<int64_t>(h) * a.nT + t];
    nv = nv < 0 ? 0 : (nv > 128 ? 128 : nv);
    nvalid_s[s] = nv;
    const uint32_t bar = smem_u32(&full_bar[s]);
    mbar_arrive_expect_tx(bar, static_cast<uint32_t>(nv) * kRowBytes);
    if (nv > 0) {
      const uint8_t* src = a.x + ((static_cast<int64_t>(b) * a.H + h) * a.nT + t) * static_cast<int64_t>(kTileBytes);
      bulk_g2s(sbase + s * kTileBytes, src, static_cast<uint32_t>(nv) * kRowBytes, bar);
    }
  };

  if (tid == 0) {
    const int64_t pro = n_local < kPoolStages ? n_local : kPoolStages;
    for (int64_t k = 0; k < pro; ++k) issue(k);
  }
  __syncthreads();   // nvalid_s of the prologue visible

  const uint32_t c16 = tid & 15, rg = tid >> 4, warp = tid >> 5, lane = tid & 31;
  for (int64_t k = 0; k < n_local; ++k) {
    const int s = static_cast<int>(k % kPoolStages);
    // thread 0 waits (bounded) and shares the verdict, so all threads leave together
    if (tid == 0) ok_s = mbar_wait(smem_u32(&full_bar[s]), static_cast<uint32_t>((k / kPoolStages) & 1), nullptr, 5);
    __syncthreads();
    if (!ok_s) {
      if (tid == 0)   // let the copies still in flight land before the CTA exits
        for (int64_t j = k + 1; j < n_local && j < k + kPoolStages; ++j)
          mbar_wait(smem_u32(&full_bar[j % kPoolStages]), static_cast<uint32_t>((j / kPoolStages) & 1), nullptr, 6);
      break;
    }
    mbar_try_wait(smem_u32(&full_bar[s]), static_cast<uint32_t>((k / kPoolStages) & 1));  // acquire
    const int32_t nv = nvalid_s[s];
    float sum[8], mx[8], mn[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) { sum[c] = 0.f; mx[c] = -INFINITY; mn[c] = INFINITY; }
    const uint8_t* buf = smem + s * kTileBytes + c16 * 16;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int32_t r = static_cast<int32_t>(rg) + 16 * i;
      if (r < nv) {
        const uint4 v = *reinterpret_cast<const uint4*>(buf + r * kRowBytes);
        const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float2 f = __bfloat1622float2(p[c]);
          sum[2 * c] += f.x; sum[2 * c + 1] += f.y;
          mx[2 * c] = fmaxf(mx[2 * c], f.x); mx[2 * c + 1] = fmaxf(mx[2 * c + 1], f.y);
          mn[2 * c] = fminf(mn[2 * c], f.x); mn[2 * c + 1] = fminf(mn[2 * c + 1], f.y);
        }
      }
    }
#pragma unroll
    for (int c = 0; c < 8; ++c) {     // lanes l and l^16 hold the same channels
      sum[c] += __shfl_xor_sync(0xffffffffu, sum[c], 16);
      mx[c] = fmaxf(mx[c], __shfl_xor_sync(0xffffffffu, mx[c], 16));
      mn[c] = fminf(mn[c], __shfl_xor_sync(0xffffffffu, mn[c], 16));
    }
    if (lane < 16) {
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        red[warp][0][c16 * 8 + c] = sum[c];
        red[warp][1][c16 * 8 + c] = mx[c];
        red[warp][2][c16 * 8 + c] = mn[c];
      }
    }
    __syncthreads();
    if (tid < 128) {
      float s0 = 0.f, m0 = -INFINITY, n0 = INFINITY;
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        s0 += red[w][0][tid];
        m0 = fmaxf(m0, red[w][1][tid]);
        n0 = fminf(n0, red[w][2][tid]);
      }
      int32_t b, h, t;
      unit_coords(first + k * stride, a.H, a.nT, b, h, t);
      float* o = a.out + (((static_cast<int64_t>(b) * a.H + h) * a.nT + t) * 3) * 128;
      if (nv > 0) {
        o[tid] = s0 / static_cast<float>(nv);
        o[128 + tid] = m0;
        o[256 + tid] = n0;
      } else {
        o[tid] = 0.f; o[128 + tid] = 0.f; o[256 + tid] = 0.f;
      }
    }
    __syncthreads();   // buffer s and red[] free again
    if (tid == 0 && k + kPoolStages < n_local) issue(k + kPoolStages);
    __syncthreads();   // nvalid_s of the refilled slot visible
  }
}

}  // namespace veda
