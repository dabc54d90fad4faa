// k_scores.cuh -- step 3: per-head residual projection of the pooled features and the
// (query tile, key tile) score matrix.
//
// "Miowtion" README, bullet "Sparse acceleration (Veda)" (a small per-head predictor
// scores (query tile, key tile) pairs) and Key Features ("mean/max/min pooling +
// per-head residual projection"):
//   qhat = mean_q + Wq[h] [mean; max; min]_q,   khat likewise,   S = qhat khat^T.
// Both products are "NT" GEMMs (both operands have K contiguous). This file holds a
// plain fp32 FFMA tiled GEMM used for both: 64 x 64 output tiles, 16-deep K slices
// staged in shared memory, 4 x 4 outputs per thread.
#pragma once

#include "veda_ptx.cuh"

namespace veda {

constexpr int kGemmBM = 64, kGemmBN = 64, kGemmBK = 16, kGemmThreads = 256;

// Batch z = ((which * B) + b) * H + h. Operand pointers:
//   A = a0[which] + (b*H + h) * a_bh,   B = b0[which] + h * b_h  (+ b * b_b),
//   R = r0[which] + (b*H + h) * r_bh (optional residual), C = c0 + z * c_z.
struct NtGemmArgs {
  const float* a0[2];
  const float* b0[2];
  const float* r0[2];
  float* c0;
  int64_t a_bh, b_h, b_b, r_bh, c_z;
  int32_t lda, ldb, ldr, ldc;
  int32_t M, N, K;
  int32_t B, H;
};

__global__ void __launch_bounds__(kGemmThreads) nt_gemm_kernel(const NtGemmArgs g) {
  __shared__ float As[kGemmBK][kGemmBM + 4];
  __shared__ float Bs[kGemmBK][kGemmBN + 4];
  const int z = blockIdx.z;
  const int h = z % g.H;
  const int b = (z / g.H) % g.B;
  const int which = z / (g.H * g.B);
  const int64_t bh = static_cast<int64_t>(b) * g.H + h;
  const float* A = g.a0[which] + bh * g.a_bh;
  const float* Bm = g.b0[which] + h * g.b_h + b * g.b_b;
  const float* R = g.r0[which] ? g.r0[which] + bh * g.r_bh : nullptr;
  float* C = g.c0 + static_cast<int64_t>(z) * g.c_z;

  const int m0 = blockIdx.y * kGemmBM, n0 = blockIdx.x * kGemmBN;
  const int tid = threadIdx.x;
  const int ty = tid / 16, tx = tid % 16;
  const int lr = tid / 4, lk = (tid % 4) * 4;   // loader: row lr, k lk..lk+3

  float acc[4][4] = {};
  for (int k0 = 0; k0 < g.K; k0 += kGemmBK) {
    float4 av = make_float4(0.f, 0.f, 0.f, 0.f), bv = av;
    if (m0 + lr < g.M && k0 + lk < g.K)
      av = *reinterpret_cast<const float4*>(A + static_cast<int64_t>(m0 + lr) * g.lda + k0 + lk);
    if (n0 + lr < g.N && k0 + lk < g.K)
      bv = *reinterpret_cast<const float4*>(Bm + static_cast<int64_t>(n0 + lr) * g.ldb + k0 + lk);
    As[lk + 0][lr] = av.x; As[lk + 1][lr] = av.y; As[lk + 2][lr] = av.z; As[lk + 3][lr] = av.w;
    Bs[lk + 0][lr] = bv.x; Bs[lk + 1][lr] = bv.y; Bs[lk + 2][lr] = bv.z; Bs[lk + 3][lr] = bv.w;
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kGemmBK; ++kk) {
      const float4 a4 = *reinterpret_cast<const float4*>(&As[kk][ty * 4]);
      const float4 b4 = *reinterpret_cast<const float4*>(&Bs[kk][tx * 4]);
      const float ar[4] = {a4.x, a4.y, a4.z, a4.w};
      const float br[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(ar[i], br[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= g.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= g.N) continue;
      float v = acc[i][j];
      if (R) v += R[static_cast<int64_t>(m) * g.ldr + n];
      C[static_cast<int64_t>(m) * g.ldc + n] = v;
    }
  }
}

}  // namespace veda
