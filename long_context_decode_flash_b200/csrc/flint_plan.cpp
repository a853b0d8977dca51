// flint_plan.cpp -- the split-KV work planner (pure host code).
//
// Work arrives as segments: one per problem (a layer, or a request), each a
// run of 32-token tiles that cover all four KV heads.  The planner lays the concatenated segments over the CTAs of one
// launch so that every CTA carries the same cost, where an item (a tile range
// of one segment on one CTA) costs its tiles plus a fixed per-item overhead
// (q set-up, merge, partial write).  Segments are cut only at CTA boundaries
// and never into pieces smaller than kMinPiece tiles, so a CTA holds a few
// items and the items of one segment sit on consecutive CTAs.
#include <stdint.h>

#include "flint.h"

namespace {
constexpr int kMinPiece = 2;
}

extern "C" int32_t flint_plan_items(const int32_t* seg_tiles, int32_t n_segs, int32_t num_ctas,
                                    int32_t item_cost, int32_t* item_seg, int32_t* item_t0,
                                    int32_t* item_t1, int32_t* cta_begin, int32_t max_items) {
  if (!seg_tiles || !item_seg || !item_t0 || !item_t1 || !cta_begin) return -1;
  if (n_segs < 1 || num_ctas < 1 || item_cost < 0 || max_items < 1) return -1;
  int64_t tiles_left = 0;
  for (int32_t s = 0; s < n_segs; ++s) {
    if (seg_tiles[s] < 1) return -1;
    tiles_left += seg_tiles[s];
  }
  int64_t segs_left = n_segs;  // segments not finished yet (the current one included)
  int32_t n = 0, c = 0;
  // Budget of CTA c: the cost still to place over the CTAs still open, where
  // every unfinished segment needs one more item and every CTA boundary still
  // ahead splits about one segment.
  auto budget = [&](int32_t cta) {
    const int64_t open = num_ctas - cta;
    const int64_t cost = tiles_left + item_cost * (segs_left + open - 1);
    return (cost + open - 1) / open;
  };
  int64_t cap = budget(0), load = 0;
  cta_begin[0] = 0;
  for (int32_t s = 0; s < n_segs; ++s) {
    const int32_t T = seg_tiles[s];
    int32_t t = 0;
    while (t < T) {
      const int64_t room = cap - load - item_cost;
      int32_t take;
      if (c == num_ctas - 1 || room >= T - t) {
        take = T - t;
      } else if (room >= kMinPiece) {
        take = static_cast<int32_t>(room);
      } else {
        ++c;  // this CTA is full: close it
        cta_begin[c] = n;
        cap = budget(c);
        load = 0;
        continue;
      }
      if (n >= max_items) return -1;
      item_seg[n] = s;
      item_t0[n] = t;
      item_t1[n] = t + take;
      ++n;
      load += take + item_cost;
      tiles_left -= take;
      t += take;
      if (t == T) --segs_left;
      if (load >= cap && c < num_ctas - 1) {
        ++c;
        cta_begin[c] = n;
        cap = budget(c);
        load = 0;
      }
    }
  }
  for (int32_t cc = c + 1; cc <= num_ctas; ++cc) cta_begin[cc] = n;
  return n;
}
