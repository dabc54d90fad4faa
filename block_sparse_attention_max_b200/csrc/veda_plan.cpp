// veda_plan.cpp -- host step of the oracle tile-plan search: the layer's vote over the
// candidate tile shapes.
//
// "Miowtion" README, Key Features / Veda sparse attention: tile shapes are chosen per
// layer by an oracle search over the relative output MSE under the best mask, by
// majority vote, with at most two shapes per layer. The errors come from the device
// (veda_rel_error, per head and candidate); the vote itself is a few comparisons per head.
//
// Reading of the vote: a head's ballot goes to its candidate of least error (the earliest
// of equal errors); the layer keeps the candidates with the most ballots, at most
// max_shapes of them and only candidates that received a ballot (the earliest of equal
// counts first); every head then takes whichever kept candidate has its least error (the
// earliest of equal errors).
#include <cmath>
#include <cstdint>
#include <string>
#include <vector>

#include "../../include/veda.h"

namespace veda {
void set_last_error(const std::string& msg);
}

extern "C" {

veda_status veda_tile_plan_vote(const double* errors, int32_t H, int32_t C, int32_t max_shapes,
                                int32_t* kept, int32_t* n_kept, int32_t* assign) {
  if (errors == nullptr || kept == nullptr || n_kept == nullptr || assign == nullptr || H < 1 || C < 1 ||
      max_shapes < 1) {
    veda::set_last_error("veda_tile_plan_vote: bad pointer or size");
    return VEDA_ERR_INVALID_ARG;
  }
  const int64_t total = static_cast<int64_t>(H) * C;
  for (int64_t i = 0; i < total; ++i)
    if (std::isnan(errors[i])) {
      veda::set_last_error("veda_tile_plan_vote: NaN error at head " + std::to_string(i / C) + ", candidate " +
                           std::to_string(i % C));
      return VEDA_ERR_INVALID_ARG;
    }
  auto err = [&](int32_t h, int32_t c) { return errors[static_cast<int64_t>(h) * C + c]; };

  std::vector<int64_t> ballots(C, 0);
  for (int32_t h = 0; h < H; ++h) {
    int32_t best = 0;
    for (int32_t c = 1; c < C; ++c)
      if (err(h, c) < err(h, best)) best = c;
    ++ballots[best];
  }
  std::vector<char> taken(C, 0);
  int32_t n = 0;
  while (n < max_shapes) {
    int32_t pick = -1;
    for (int32_t c = 0; c < C; ++c)
      if (!taken[c] && ballots[c] > 0 && (pick < 0 || ballots[c] > ballots[pick])) pick = c;
    if (pick < 0) break;
    taken[pick] = 1;
    ++n;
  }
  int32_t m = 0;
  for (int32_t c = 0; c < C; ++c)
    if (taken[c]) kept[m++] = c;
  *n_kept = n;
  for (int32_t h = 0; h < H; ++h) {
    int32_t best = kept[0];
    for (int32_t i = 1; i < n; ++i)
      if (err(h, kept[i]) < err(h, best)) best = kept[i];
    assign[h] = best;
  }
  return VEDA_OK;
}

}  // extern "C"
