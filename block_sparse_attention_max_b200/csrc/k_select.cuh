// k_select.cuh -- step 4: per-row block lists under Bresenham budgets with a forced
// diagonal, split into full and partial key tiles.
//
// "Miowtion" README, Key Features / Veda sparse attention: equal-kernel-cost budgets
// with Bresenham rounding, forced diagonal tiles, segmented reference/target budgets,
// full/partial block lists.
//
// One warp per (batch, head, query row). Each candidate key tile j gets a 32-bit rank
// image u_j of its score (order-preserving, complemented so that the highest score has
// the smallest image, -0 folded onto +0, NaN last); the diagonal gets u = 0, below any
// real score. For every segment s the k_s-th smallest image T_s is found by a radix
// select (four 8-bit digits, most significant first, one shared-memory histogram per
// segment and digit). The row then takes every tile with u < T_s and, among the tiles
// with u == T_s, the lowest indices until k_s are taken -- exactly "score descending,
// ties to the lower index". Selected tiles are written in ascending index order by
// ballot compaction, into the full list (tile_valid == 128) or the partial list.
#pragma once

#include "veda_ptx.cuh"

namespace veda {

constexpr int kSelWarps = 8;                   // query rows per CTA
constexpr int kSelThreads = 32 * kSelWarps;
constexpr int kSelMaxTiles = 2048;
constexpr int kMaxSeg = 4;

// Shared memory of one warp, sized to the launch's tile count and segments (so that short
// rows leave room for more resident warps): rank images [nT], segment ids [nT] (bytes,
// rounded to 16), one 256-bin histogram per segment.
__host__ __device__ constexpr uint32_t sel_warp_bytes(int32_t nT, int32_t n_seg) {
  return static_cast<uint32_t>(nT) * 4u + ((static_cast<uint32_t>(nT) + 15u) & ~15u) +
         static_cast<uint32_t>(n_seg) * 1024u;
}
constexpr uint32_t kSelMaxSmem = kSelWarps * sel_warp_bytes(kSelMaxTiles, kMaxSeg);

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

// Order-preserving map of fp32 onto uint32 (ascending), complemented so that the highest
// score has the smallest image; -0 is folded onto +0 and NaN ranks last.
__device__ __forceinline__ uint32_t score_rank_bits(float f, bool& is_nan) {
  is_nan = f != f;
  if (is_nan) return 0xFFFFFFFFu;
  if (f == 0.0f) f = 0.0f;
  uint32_t u = __float_as_uint(f);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ~u;   // +inf -> 0x007FFFFF; never 0
}

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

__global__ void __launch_bounds__(kSelThreads) select_kernel(const SelectArgs a) {
  extern __shared__ __align__(16) uint8_t sel_smem[];
  const int w = threadIdx.x >> 5;
  uint8_t* wbase = sel_smem + static_cast<uint32_t>(w) * sel_warp_bytes(a.nT, a.n_seg);
  uint32_t* su = reinterpret_cast<uint32_t*>(wbase);
  uint8_t* ss = wbase + static_cast<uint32_t>(a.nT) * 4u;
  uint32_t* hist = reinterpret_cast<uint32_t*>(ss + ((static_cast<uint32_t>(a.nT) + 15u) & ~15u));
  const uint32_t lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kSelWarps + w;
  if (row >= static_cast<int64_t>(a.B) * a.H * a.nT) return;
  const int32_t r = static_cast<int32_t>(row % a.nT);
  const int32_t h = static_cast<int32_t>((row / a.nT) % a.H);
  int32_t n = a.nT_per_head[h];
  if (n < 0 || n > a.nT) {
    if (lane == 0) flag_status(ST_BAD_LIST);
    n = 0;
  }
  if (r >= n) {            // past the head's tiles: empty lists
    if (lane == 0) { a.full_cnt[row] = 0; a.part_cnt[row] = 0; }
    return;
  }
  const int32_t nseg = a.n_seg;
  const int32_t* seg_h = a.segment + static_cast<int64_t>(h) * a.nT;
  const int32_t* val_h = a.valid + static_cast<int64_t>(h) * a.nT;
  const float* srow = a.scores + row * a.nT;

  // candidates -> shared memory; tiles per segment
  int32_t cnt[kMaxSeg] = {0, 0, 0, 0};
  bool saw_nan = false, bad_seg = false;
  for (int32_t j = static_cast<int32_t>(lane); j < n; j += 32) {
    int32_t sg = seg_h[j];
    if (sg < 0 || sg >= nseg) { bad_seg = true; sg = nseg - 1; }
    bool nan = false;
    uint32_t u = score_rank_bits(srow[j], nan);
    saw_nan |= nan;
    if (j == r) u = 0;
    su[j] = u;
    ss[j] = static_cast<uint8_t>(sg);
#pragma unroll
    for (int s = 0; s < kMaxSeg; ++s) cnt[s] += (sg == s);
  }
  if (saw_nan) flag_status(ST_NAN_SCORE);
  if (bad_seg) flag_status(ST_BAD_LIST);
  int32_t own = seg_h[r];
  if (own < 0 || own >= nseg) own = nseg - 1;

  // budgets of this row (exact integer Bresenham per segment)
  int32_t k[kMaxSeg], krem[kMaxSeg];
  uint32_t prefix[kMaxSeg];
#pragma unroll
  for (int s = 0; s < kMaxSeg; ++s) {
    int32_t nK = cnt[s];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) nK += __shfl_xor_sync(0xffffffffu, nK, o);
    int64_t kk = 0;
    if (s < nseg) {
      const int64_t num = static_cast<int64_t>(nK) * a.rho_num[s];
      kk = ((r + 1) * num) / a.rho_den[s] - (static_cast<int64_t>(r) * num) / a.rho_den[s];
      if (s == own && kk < 1) kk = 1;
      if (kk > nK) kk = nK;
      if (kk < 0) kk = 0;
    }
    k[s] = static_cast<int32_t>(kk);
    krem[s] = k[s];
    prefix[s] = 0;
  }
  __syncwarp();

  // radix select of the k_s-th smallest image per segment
  for (int d = 3; d >= 0; --d) {
    const int shift = 8 * d;
    const uint32_t hi_mask = d == 3 ? 0u : (0xFFFFFFFFu << (shift + 8));
    for (int i = static_cast<int>(lane); i < nseg * 256; i += 32) hist[i] = 0;
    __syncwarp();
    for (int32_t j = static_cast<int32_t>(lane); j < n; j += 32) {
      const uint32_t u = su[j];
      const int sg = ss[j];
      if (k[sg] > 0 && (u & hi_mask) == prefix[sg]) atomicAdd(&hist[sg * 256 + ((u >> shift) & 255u)], 1u);
    }
    __syncwarp();
#pragma unroll
    for (int s = 0; s < kMaxSeg; ++s) {
      if (s >= nseg || k[s] == 0) continue;       // warp-uniform
      uint32_t c8[8];
      uint32_t local = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) { c8[i] = hist[s * 256 + lane * 8 + i]; local += c8[i]; }
      uint32_t incl = local;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t x = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= static_cast<uint32_t>(o)) incl += x;
      }
      uint32_t before = incl - local;
      int found_bin = -1;
      uint32_t found_before = 0;
      const uint32_t want = static_cast<uint32_t>(krem[s]);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (found_bin < 0 && before < want && want <= before + c8[i]) {
          found_bin = static_cast<int>(lane * 8 + i);
          found_before = before;
        }
        before += c8[i];
      }
      const uint32_t who = __ballot_sync(0xffffffffu, found_bin >= 0);
      const int src = who ? __ffs(who) - 1 : 0;
      found_bin = __shfl_sync(0xffffffffu, found_bin, src);
      found_before = __shfl_sync(0xffffffffu, found_before, src);
      if (found_bin >= 0) {
        prefix[s] |= static_cast<uint32_t>(found_bin) << shift;
        krem[s] -= static_cast<int32_t>(found_before);
      }
    }
    __syncwarp();
  }

  // selection and ascending compaction (chunks of 32 tiles in index order)
  int32_t eq_taken[kMaxSeg] = {0, 0, 0, 0};
  int32_t nf = 0, np = 0;
  int32_t* fo = a.full_idx + row * a.stride;
  int32_t* po = a.part_idx + row * a.stride;
  const uint32_t lt = lanemask_lt();
  for (int32_t j0 = 0; j0 < n; j0 += 32) {
    const int32_t j = j0 + static_cast<int32_t>(lane);
    const bool in = j < n;
    const int sg = in ? ss[j] : 0;
    const uint32_t u = in ? su[j] : 0xFFFFFFFFu;
    const bool take_seg = in && k[sg] > 0;
    const bool less = take_seg && u < prefix[sg];
    const bool eq = take_seg && u == prefix[sg];
    int32_t rank = 0;
    bool sel = less;
#pragma unroll
    for (int s = 0; s < kMaxSeg; ++s) {
      const uint32_t be = __ballot_sync(0xffffffffu, eq && sg == s);
      if (eq && sg == s) {
        rank = eq_taken[s] + __popc(be & lt);
        sel = rank < krem[s];
      }
      eq_taken[s] += __popc(be);
    }
    const bool full = sel && val_h[in ? j : 0] == 128;
    const bool part = sel && !full;
    const uint32_t bf = __ballot_sync(0xffffffffu, full);
    const uint32_t bp = __ballot_sync(0xffffffffu, part);
    if (full) { const int32_t p = nf + __popc(bf & lt); if (p < a.stride) fo[p] = j; }
    if (part) { const int32_t p = np + __popc(bp & lt); if (p < a.stride) po[p] = j; }
    nf += __popc(bf);
    np += __popc(bp);
  }
  if (lane == 0) {
    if (nf > a.stride || np > a.stride) flag_status(ST_LIST_OVERFLOW);
    a.full_cnt[row] = nf < a.stride ? nf : a.stride;
    a.part_cnt[row] = np < a.stride ? np : a.stride;
  }
}

}  // namespace veda
