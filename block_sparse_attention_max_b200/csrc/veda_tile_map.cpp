// veda_tile_map.cpp -- host construction of the per-head slot -> raster-token map.
//
// "Miowtion" README, bullet "Sparse acceleration (Veda)": video tokens are permuted
// into 3D tiles of 128 tokens. Key Features / Veda sparse attention: up to two
// (t, h, w) tile shapes per layer (per head), padded grids with valid-prefix tiles,
// segmented reference/target budgets. NEWS 2026/09/23: per-head dynamic tile
// permutations.
//
// Layout produced (see veda.h): for each head the grid is padded up to a multiple of
// the head's tile shape, tiles are enumerated in raster order of tile coordinates
// (then reordered by the optional per-head tile order), the valid tokens of a tile
// fill its first slots in local (t, h, w) raster order and the rest are pads (-1).
// Appended 1D tokens follow as 1D tiles of 128 in key segment 1.
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <string>
#include <vector>

#include "../../include/veda.h"

namespace veda {
void set_last_error(const std::string& msg);
}

namespace {

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

bool shape_ok(const veda_tile_shape& s) {
  return s.t > 0 && s.h > 0 && s.w > 0 && static_cast<int64_t>(s.t) * s.h * s.w == VEDA_TILE;
}

int64_t video_tiles(const veda_geometry& g, const veda_tile_shape& s) {
  if (static_cast<int64_t>(g.T) * g.Hg * g.Wg == 0) return 0;
  return ceil_div(g.T, s.t) * ceil_div(g.Hg, s.h) * ceil_div(g.Wg, s.w);
}

veda_status check_geometry(const veda_geometry* g) {
  if (g == nullptr || g->head_shape == nullptr || g->H <= 0 || g->T < 0 || g->Hg < 0 ||
      g->Wg < 0 || g->n_tail < 0) {
    veda::set_last_error("geometry: NULL pointer or negative size");
    return VEDA_ERR_INVALID_ARG;
  }
  for (int32_t h = 0; h < g->H; ++h) {
    if (!shape_ok(g->head_shape[h])) {
      veda::set_last_error("geometry: tile shape of head " + std::to_string(h) +
                           " does not hold 128 tokens");
      return VEDA_ERR_INVALID_ARG;
    }
  }
  const int64_t N = static_cast<int64_t>(g->T) * g->Hg * g->Wg + g->n_tail;
  if (N > INT32_MAX || N == 0) {
    veda::set_last_error("geometry: token count out of range");
    return VEDA_ERR_INVALID_ARG;
  }
  if (g->tile_order != nullptr) {
    int64_t need = 0;
    for (int32_t h = 0; h < g->H; ++h) need = std::max(need, video_tiles(*g, g->head_shape[h]));
    if (g->order_stride < need) {
      veda::set_last_error("geometry: order_stride smaller than the video tile count");
      return VEDA_ERR_INVALID_ARG;
    }
  }
  return VEDA_OK;
}

}  // namespace

extern "C" veda_status veda_geometry_sizes(const veda_geometry* g, int32_t* N, int32_t* nT_max,
                                           int32_t* Npad_max) {
  veda_status st = check_geometry(g);
  if (st != VEDA_OK) return st;
  const int64_t tail_tiles = ceil_div(g->n_tail, VEDA_TILE);
  int64_t nt = 0;
  for (int32_t h = 0; h < g->H; ++h)
    nt = std::max(nt, video_tiles(*g, g->head_shape[h]) + tail_tiles);
  if (nt * VEDA_TILE > INT32_MAX) {
    veda::set_last_error("geometry: padded slot count out of range");
    return VEDA_ERR_INVALID_ARG;
  }
  if (N) *N = static_cast<int32_t>(static_cast<int64_t>(g->T) * g->Hg * g->Wg + g->n_tail);
  if (nT_max) *nT_max = static_cast<int32_t>(nt);
  if (Npad_max) *Npad_max = static_cast<int32_t>(nt * VEDA_TILE);
  return VEDA_OK;
}

extern "C" veda_status veda_build_tile_map(const veda_geometry* g, int32_t* tile_map,
                                           int32_t* tile_valid, int32_t* tile_segment,
                                           int32_t* nT_per_head) {
  int32_t N = 0, nT = 0, Npad = 0;
  veda_status st = veda_geometry_sizes(g, &N, &nT, &Npad);
  if (st != VEDA_OK) return st;
  if (!tile_map || !tile_valid || !tile_segment || !nT_per_head) {
    veda::set_last_error("veda_build_tile_map: NULL output");
    return VEDA_ERR_INVALID_ARG;
  }
  const int64_t n_video = static_cast<int64_t>(g->T) * g->Hg * g->Wg;
  for (int32_t h = 0; h < g->H; ++h) {
    const veda_tile_shape s = g->head_shape[h];
    int32_t* map = tile_map + static_cast<int64_t>(h) * Npad;
    int32_t* valid = tile_valid + static_cast<int64_t>(h) * nT;
    int32_t* seg = tile_segment + static_cast<int64_t>(h) * nT;
    std::fill(map, map + Npad, -1);
    std::fill(valid, valid + nT, 0);
    std::fill(seg, seg + nT, 0);

    const int64_t nvt = video_tiles(*g, s);
    const int64_t gt = n_video ? ceil_div(g->T, s.t) : 0;
    const int64_t gh = n_video ? ceil_div(g->Hg, s.h) : 0;
    const int64_t gw = n_video ? ceil_div(g->Wg, s.w) : 0;
    // validate the per-head order: a permutation of [0, nvt)
    const int32_t* order = g->tile_order ? g->tile_order + static_cast<int64_t>(h) * g->order_stride
                                         : nullptr;
    if (order) {
      std::vector<char> seen(static_cast<size_t>(nvt), 0);
      for (int64_t p = 0; p < nvt; ++p) {
        if (order[p] < 0 || order[p] >= nvt || seen[order[p]]) {
          veda::set_last_error("geometry: tile_order of head " + std::to_string(h) +
                               " is not a permutation");
          return VEDA_ERR_INVALID_ARG;
        }
        seen[order[p]] = 1;
      }
    }
    for (int64_t p = 0; p < nvt; ++p) {
      const int64_t tile = order ? order[p] : p;   // raster tile index placed at position p
      const int64_t it = tile / (gh * gw), ih = (tile / gw) % gh, iw = tile % gw;
      int32_t n = 0;
      int32_t* dst = map + p * VEDA_TILE;
      for (int32_t lt = 0; lt < s.t; ++lt) {
        const int64_t t = it * s.t + lt;
        if (t >= g->T) break;
        for (int32_t lh = 0; lh < s.h; ++lh) {
          const int64_t y = ih * s.h + lh;
          if (y >= g->Hg) break;
          for (int32_t lw = 0; lw < s.w; ++lw) {
            const int64_t x = iw * s.w + lw;
            if (x >= g->Wg) break;
            dst[n++] = static_cast<int32_t>((t * g->Hg + y) * g->Wg + x);
          }
        }
      }
      valid[p] = n;
      seg[p] = 0;
    }
    (void)gt;
    const int64_t tail_tiles = ceil_div(g->n_tail, VEDA_TILE);
    for (int64_t q = 0; q < tail_tiles; ++q) {
      const int64_t p = nvt + q;
      const int64_t j0 = q * VEDA_TILE;
      const int64_t n = std::min<int64_t>(VEDA_TILE, g->n_tail - j0);
      for (int64_t i = 0; i < n; ++i) map[p * VEDA_TILE + i] = static_cast<int32_t>(n_video + j0 + i);
      valid[p] = static_cast<int32_t>(n);
      seg[p] = 1;
    }
    nT_per_head[h] = static_cast<int32_t>(nvt + tail_tiles);
  }
  return VEDA_OK;
}
