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

// ---- static lists plus a run-time queue --------------------------------------
//
// A static plan fixes every CTA's work before the launch, but CTAs do not
// stream at the same rate (on B200 a fixed set of SMs reads ~10 % slower than
// the rest while all of them stream), so the fast ones idle at the end.  Here
// each large segment keeps only its first ~80 % of tiles in the static plan;
// its tail is cut into chunks that CTAs claim from a shared queue once their
// static lists are done.  Chunk sizes follow guided self-scheduling over the
// whole pool (ceil(remaining / CTAs), never below a floor), so early claims are
// large and the last ones small.  Chunk boundaries are fixed here, on the host:
// every item is computed the same way whichever CTA claims it, and partials
// are merged in item order, so results stay bitwise deterministic.

#include <algorithm>
#include <vector>

namespace {

#ifndef FLINT_DYN_MIN_TILES
#define FLINT_DYN_MIN_TILES 64
#endif
#ifndef FLINT_DYN_MIN_SHARE
#define FLINT_DYN_MIN_SHARE 64
#endif
#ifndef FLINT_DYN_SMALL_PERMILLE
#define FLINT_DYN_SMALL_PERMILLE 200
#endif
#ifndef FLINT_DYN_SMALL_CHUNK
#define FLINT_DYN_SMALL_CHUNK 8
#endif
constexpr int kDynMinTiles = FLINT_DYN_MIN_TILES;  // smaller segments stay wholly static
// Below this many tiles per CTA the whole launch stays static: a CTA's share
// is then short next to a chunk, and the few SMs that stream slower cost less
// than the queue's extra items.
constexpr int kDynMinShare = FLINT_DYN_MIN_SHARE;

struct Variant {
  int permille;   // share of a large segment's tiles put in the queue
  int chunk_min;  // smallest chunk, tiles
};
// Tried in order until the plan fits max_items; the last one is static only.
// A variant whose smallest chunk exceeds an eighth of a CTA's share is
// skipped: a chunk that large taken late would itself be the tail.  The
// variant before the static one serves short shares (few tiles per CTA).
constexpr Variant kVariants[] = {{200, 8},
                                 {200, 16},
                                 {200, 32},
                                 {100, 32},
                                 {FLINT_DYN_SMALL_PERMILLE, FLINT_DYN_SMALL_CHUNK},
                                 {0, 0}};

}  // namespace

extern "C" int32_t flint_plan_split(const int32_t* seg_tiles, int32_t n_segs, int32_t num_ctas,
                                    int32_t item_cost, int32_t max_items, int32_t* item_seg,
                                    int32_t* item_t0, int32_t* item_t1, int32_t* order,
                                    int32_t* cta_begin) {
  if (!seg_tiles || !item_seg || !item_t0 || !item_t1 || !order || !cta_begin) return -1;
  if (n_segs < 1 || num_ctas < 1 || item_cost < 0 || max_items < 1) return -1;
  int64_t total = 0;
  for (int32_t s = 0; s < n_segs; ++s) {
    if (seg_tiles[s] < 1) return -1;
    total += seg_tiles[s];
  }
  const bool queue_pays = total >= static_cast<int64_t>(kDynMinShare) * num_ctas;
  std::vector<int32_t> st(n_segs), ss(max_items), s0(max_items), s1(max_items);
  struct Piece {
    int32_t seg, t0, t1, rank;  // rank: position in the static lists, or kQueue + queue position
  };
  constexpr int32_t kQueue = 1 << 20;
  for (const Variant& v : kVariants) {
    if (v.permille > 0 && (!queue_pays || static_cast<int64_t>(v.chunk_min) * 8 * num_ctas > total)) continue;
    int64_t pool = 0;
    for (int32_t s = 0; s < n_segs; ++s) {
      const int32_t d = (v.permille > 0 && seg_tiles[s] >= kDynMinTiles)
                            ? static_cast<int32_t>(static_cast<int64_t>(seg_tiles[s]) * v.permille / 1000)
                            : 0;
      st[s] = seg_tiles[s] - d;
      pool += d;
    }
    const int32_t ns = flint_plan_items(st.data(), n_segs, num_ctas, item_cost, ss.data(), s0.data(),
                                        s1.data(), cta_begin, max_items);
    if (ns < 0) continue;
    std::vector<Piece> pieces;
    pieces.reserve(max_items);
    for (int32_t i = 0; i < ns; ++i) pieces.push_back({ss[i], s0[i], s1[i], i});
    // the queue: guided chunk sizes, taken round robin from the segments' tails
    std::vector<int32_t> next(st);
    int64_t rem = pool;
    int32_t rr = 0, q = 0;
    bool fits = true;
    while (rem > 0) {
      if (static_cast<int32_t>(pieces.size()) >= max_items) {
        fits = false;
        break;
      }
      const int64_t want = std::max<int64_t>(v.chunk_min, (rem + num_ctas - 1) / num_ctas);
      while (next[rr] >= seg_tiles[rr]) rr = (rr + 1) % n_segs;
      const int32_t take = static_cast<int32_t>(std::min<int64_t>(want, seg_tiles[rr] - next[rr]));
      pieces.push_back({rr, next[rr], next[rr] + take, kQueue + q++});
      next[rr] += take;
      rem -= take;
      rr = (rr + 1) % n_segs;
    }
    if (!fits) continue;
    // items sorted by (segment, first tile): a segment's static items come
    // first, then its queued chunks, all in tile order
    std::vector<int32_t> idx(pieces.size());
    for (size_t i = 0; i < idx.size(); ++i) idx[i] = static_cast<int32_t>(i);
    std::sort(idx.begin(), idx.end(), [&](int32_t a, int32_t b) {
      return pieces[a].seg != pieces[b].seg ? pieces[a].seg < pieces[b].seg : pieces[a].t0 < pieces[b].t0;
    });
    for (size_t k = 0; k < idx.size(); ++k) {
      const Piece& p = pieces[idx[k]];
      item_seg[k] = p.seg;
      item_t0[k] = p.t0;
      item_t1[k] = p.t1;
      order[p.rank < kQueue ? p.rank : ns + (p.rank - kQueue)] = static_cast<int32_t>(k);
    }
    return static_cast<int32_t>(pieces.size());
  }
  return -1;
}
