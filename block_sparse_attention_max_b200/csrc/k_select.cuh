// k_select.cuh -- step 4: per-row block lists under Bresenham budgets with a forced
// diagonal, split into full and partial key tiles.
//
// "Miowtion" README, Key Features / Veda sparse attention: equal-kernel-cost budgets
// with Bresenham rounding, forced diagonal tiles, segmented reference/target budgets,
// full/partial block lists. One CTA per (batch, head, query row). Every candidate key
// tile gets one 64-bit key that orders it within its segment:
//   bits 48..51  segment
//   bits 16..47  descending-order image of the fp32 score (-0 folded onto +0);
//                0 is reserved for the diagonal, which therefore comes first
//   bits  0..15  tile index (equal scores: lower index first)
// After an ascending bitonic sort the k-th key of each segment is that segment's
// threshold; a tile is selected when its key is at or below its segment's threshold.
// Selected tiles are compacted in ascending index order.
#pragma once

#include "veda_ptx.cuh"

namespace veda {

constexpr int kSelThreads = 512;
constexpr int kSelMaxTiles = 2048;
constexpr int kSelPerThread = kSelMaxTiles / kSelThreads;   // 4
constexpr int kMaxSeg = 4;

struct SelectArgs {
  const float* scores;          // [B][H][nT][nT]
  const int32_t* valid;         // [H][nT]
  const int32_t* segment;       // [H][nT]
  const int32_t* nT_per_head;   // [H]
  int32_t* full_cnt;            // [B][H][nT]
  int32_t* full_idx;            // [B][H][nT][stride]
  int32_t* part_cnt;
  int32_t* part_idx;
  int32_t stride, B, H, nT, n_seg;
  int32_t rho_num[kMaxSeg], rho_den[kMaxSeg];
};

// Order-preserving map of fp32 onto uint32 (ascending), then complemented so that the
// highest score has the smallest image. -0 is folded onto +0; NaN ranks last.
__device__ __forceinline__ uint32_t score_rank_bits(float f, bool& is_nan) {
  is_nan = f != f;
  if (is_nan) return 0xFFFFFFFFu;
  if (f == 0.0f) f = 0.0f;
  uint32_t u = __float_as_uint(f);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ~u;   // +inf -> 0x007FFFFF; never 0
}

__global__ void __launch_bounds__(kSelThreads, 1) select_kernel(const SelectArgs a) {
  __shared__ uint64_t keys[kSelMaxTiles];
  __shared__ int32_t seg_count[kMaxSeg];
  __shared__ int32_t warp_tot[2][kSelThreads / 32];

  const int32_t r = blockIdx.x % a.nT;
  const int32_t bh = blockIdx.x / a.nT;
  const int32_t h = bh % a.H;
  const int32_t tid = threadIdx.x;
  const int64_t row = static_cast<int64_t>(bh) * a.nT + r;
  int32_t n = a.nT_per_head[h];
  if (n < 0 || n > a.nT) {
    if (tid == 0) flag_status(ST_BAD_LIST);
    n = 0;
  }
  if (r >= n) {           // past the head's tiles: empty lists
    if (tid == 0) { a.full_cnt[row] = 0; a.part_cnt[row] = 0; }
    return;
  }
  const int32_t* seg_h = a.segment + static_cast<int64_t>(h) * a.nT;
  const int32_t* val_h = a.valid + static_cast<int64_t>(h) * a.nT;
  const float* srow = a.scores + row * a.nT;

  if (tid < kMaxSeg) seg_count[tid] = 0;
  __syncthreads();

  // keys of this thread's tiles (contiguous block of kSelPerThread tiles)
  int P = 1;
  while (P < n) P <<= 1;
  uint64_t mykey[kSelPerThread];
  int32_t myseg[kSelPerThread];
  int32_t local_cnt[kMaxSeg] = {0, 0, 0, 0};
  bool saw_nan = false;
#pragma unroll
  for (int i = 0; i < kSelPerThread; ++i) {
    const int32_t j = tid * kSelPerThread + i;
    mykey[i] = ~0ull;
    myseg[i] = -1;
    if (j < n) {
      int32_t sg = seg_h[j];
      if (sg < 0 || sg >= a.n_seg) { flag_status(ST_BAD_LIST); sg = a.n_seg - 1; }
      myseg[i] = sg;
      bool nan = false;
      uint32_t rank = score_rank_bits(srow[j], nan);
      saw_nan |= nan;
      if (j == r) rank = 0;
      mykey[i] = (static_cast<uint64_t>(sg) << 48) | (static_cast<uint64_t>(rank) << 16) |
                 static_cast<uint64_t>(j);
#pragma unroll
      for (int s = 0; s < kMaxSeg; ++s) local_cnt[s] += (sg == s);
    }
    if (j < P) keys[j] = mykey[i];
  }
  if (saw_nan) flag_status(ST_NAN_SCORE);
#pragma unroll
  for (int s = 0; s < kMaxSeg; ++s)
    if (local_cnt[s]) atomicAdd(&seg_count[s], local_cnt[s]);
  __syncthreads();

  // ascending bitonic sort of keys[0, P)
  for (int k = 2; k <= P; k <<= 1) {
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      for (int i = tid; i < P; i += kSelThreads) {
        const int l = i ^ jj;
        if (l > i) {
          const uint64_t x = keys[i], y = keys[l];
          const bool up = (i & k) == 0;
          if ((x > y) == up) { keys[i] = y; keys[l] = x; }
        }
      }
      __syncthreads();
    }
  }

  // budgets of this row (exact integer Bresenham), threshold key per segment: the keys
  // of segment s occupy sorted positions [start_s, start_s + nK_s)
  const int32_t own = seg_h[r] < 0 || seg_h[r] >= a.n_seg ? a.n_seg - 1 : seg_h[r];
  uint64_t thr[kMaxSeg];
  int32_t budget[kMaxSeg];
  int32_t start = 0;
#pragma unroll
  for (int s = 0; s < kMaxSeg; ++s) {
    thr[s] = 0;
    budget[s] = 0;
    if (s < a.n_seg) {
      const int64_t nK = seg_count[s];
      const int64_t num = nK * a.rho_num[s];
      int64_t kk = ((r + 1) * num) / a.rho_den[s] - (static_cast<int64_t>(r) * num) / a.rho_den[s];
      if (s == own && kk < 1) kk = 1;
      if (kk > nK) kk = nK;
      if (kk < 0) kk = 0;
      budget[s] = static_cast<int32_t>(kk);
      if (kk > 0) thr[s] = keys[start + kk - 1];
      start += static_cast<int32_t>(nK);
    }
  }

  // selection flags: a tile is taken when its key ranks within its segment's budget
  int32_t nf = 0, np = 0;
  bool selF[kSelPerThread], selP[kSelPerThread];
#pragma unroll
  for (int i = 0; i < kSelPerThread; ++i) {
    const int32_t j = tid * kSelPerThread + i;
    bool sel = false;
    if (j < n) {
      const int32_t sg = myseg[i];
      sel = budget[sg] > 0 && mykey[i] <= thr[sg];
    }
    const bool full = sel && val_h[j] == 128;
    selF[i] = full;
    selP[i] = sel && !full;
    nf += selF[i];
    np += selP[i];
  }
  // block-wide exclusive scan of (nf, np) in thread order
  const int lane = tid & 31, warp = tid >> 5;
  int32_t sf = nf, sp = np;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t xf = __shfl_up_sync(0xffffffffu, sf, o);
    const int32_t xp = __shfl_up_sync(0xffffffffu, sp, o);
    if (lane >= o) { sf += xf; sp += xp; }
  }
  if (lane == 31) { warp_tot[0][warp] = sf; warp_tot[1][warp] = sp; }
  __syncthreads();
  int32_t basef = 0, basep = 0, totf = 0, totp = 0;
  for (int w = 0; w < kSelThreads / 32; ++w) {
    if (w < warp) { basef += warp_tot[0][w]; basep += warp_tot[1][w]; }
    totf += warp_tot[0][w];
    totp += warp_tot[1][w];
  }
  int32_t pf = basef + sf - nf, pp = basep + sp - np;
  int32_t* fo = a.full_idx + row * a.stride;
  int32_t* po = a.part_idx + row * a.stride;
#pragma unroll
  for (int i = 0; i < kSelPerThread; ++i) {
    const int32_t j = tid * kSelPerThread + i;
    if (selF[i]) { if (pf < a.stride) fo[pf] = j; ++pf; }
    if (selP[i]) { if (pp < a.stride) po[pp] = j; ++pp; }
  }
  if (tid == 0) {
    if (totf > a.stride || totp > a.stride) flag_status(ST_LIST_OVERFLOW);
    a.full_cnt[row] = totf < a.stride ? totf : a.stride;
    a.part_cnt[row] = totp < a.stride ? totp : a.stride;
  }
}

}  // namespace veda
