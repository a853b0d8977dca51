// flint_abi.cu -- the extern "C" entry points of libflint.so: argument
// validation, split planning, TMA tensor maps and launches.  No entry point
// allocates, frees or synchronises; everything is queued on the caller's
// stream.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <cmath>
#include <mutex>
#include <string>
#include <unordered_map>
#include <vector>

#include "flint_internal.h"

using namespace flint;

namespace {

thread_local std::string g_last_error;

flint_status fail(flint_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

flint_status ok() {
  g_last_error.clear();
  return FLINT_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int kItemCost = 2;  // per-item overhead in tile units (planner cost model)

// ---- device properties (cached per device) --------------------------------

int device_num_sms(int* out) {
  static std::mutex mu;
  static int sms[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -1;
  std::lock_guard<std::mutex> lock(mu);
  if (sms[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
      return -1;
    sms[dev] = v;
  }
  *out = sms[dev];
  return 0;
}

// ---- TMA tensor maps --------------------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Encoded maps are kept per (device, base, geometry): a decode loop calls with
// the same caches every token, so encoding happens once.
struct MapKey {
  int dev;
  uintptr_t base;
  int64_t d2, d3, stride2;
  int dtype;
  bool operator==(const MapKey& o) const {
    return dev == o.dev && base == o.base && d2 == o.d2 && d3 == o.d3 && stride2 == o.stride2 &&
           dtype == o.dtype;
  }
};
struct MapKeyHash {
  size_t operator()(const MapKey& k) const {
    size_t h = std::hash<uintptr_t>()(k.base);
    h ^= std::hash<int64_t>()(k.d2 * 1000003 + k.d3) + 0x9e3779b97f4a7c15ull + (h << 6) + (h >> 2);
    h ^= std::hash<int64_t>()(k.stride2 * 31 + k.dev * 2 + k.dtype) + 0x9e3779b97f4a7c15ull + (h << 6) + (h >> 2);
    return h;
  }
};

// A K or V cache seen as a 4-D tensor (dims innermost first):
//   CONTIGUOUS/RING: [128 dims][4 heads][capacity tokens][B requests]
//   PAGED:           [128 dims][4 heads][64 tokens][num_blocks]
// read with the 128-byte swizzle in boxes of 64 dims x 1 head x kTile (32)
// tokens x 1 for bf16, and of 128 dims x 1 head x 64 tokens x 1 for E4M3
// (one byte per value); either way a box row is 128 bytes.
flint_status encode_cache_map(CUtensorMap* map, void* base, const flint_kv_cache& c, int B) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(FLINT_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const bool fp8 = c.dtype == FLINT_KV_FP8_E4M3;
  const cuuint64_t eb = fp8 ? 1 : 2;  // bytes per element
  cuuint64_t dims[4], strides[3];
  dims[0] = kDim;
  dims[1] = kKvHeads;
  strides[0] = kDim * eb;
  strides[1] = kKvHeads * kDim * eb;
  if (c.layout == FLINT_KV_PAGED) {
    dims[2] = kBlock;
    dims[3] = static_cast<cuuint64_t>(c.num_blocks);
    strides[2] = static_cast<cuuint64_t>(kBlock) * kKvHeads * kDim * eb;
  } else {
    const int64_t rs = c.req_stride ? c.req_stride : static_cast<int64_t>(c.capacity) * kKvHeads * kDim;
    dims[2] = static_cast<cuuint64_t>(c.capacity);
    dims[3] = static_cast<cuuint64_t>(B);
    strides[2] = static_cast<cuuint64_t>(rs) * eb;
  }
  static std::mutex mu;
  static std::unordered_map<MapKey, CUtensorMap, MapKeyHash> cache;
  int dev = 0;
  cudaGetDevice(&dev);
  const MapKey key{dev, reinterpret_cast<uintptr_t>(base), static_cast<int64_t>(dims[2]),
                   static_cast<int64_t>(dims[3]), static_cast<int64_t>(strides[2]), c.dtype};
  {
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end()) {
      *map = it->second;
      return FLINT_OK;
    }
  }
  const cuuint32_t box[4] = {fp8 ? static_cast<cuuint32_t>(kDim) : 64u, 1,
                            static_cast<cuuint32_t>(fp8 ? kTileFp8 : kTile), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base, dims,
                  strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  static_cast<CUtensorMapL2promotion>(FLINT_L2_PROMOTION),
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FLINT_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
  std::lock_guard<std::mutex> lock(mu);
  if (cache.size() >= 4096) cache.clear();
  cache.emplace(key, *map);
  return FLINT_OK;
}

// ---- validation -------------------------------------------------------------

flint_status check_cache(const flint_kv_cache* c, int B, const char* who) {
  if (!c) return fail(FLINT_ERR_INVALID_ARG, "%s: cache is NULL", who);
  if (!c->k || !c->v) return fail(FLINT_ERR_INVALID_ARG, "%s: cache k/v is NULL", who);
  if (c->dtype != FLINT_KV_BF16 && c->dtype != FLINT_KV_FP8_E4M3)
    return fail(FLINT_ERR_INVALID_ARG, "%s: unknown cache dtype %d", who, c->dtype);
  if (c->dtype == FLINT_KV_FP8_E4M3)
    for (int g = 0; g < kKvHeads; ++g)
      if (!(c->k_scale[g] > 0.f && c->k_scale[g] < 3.0e38f) || !(c->v_scale[g] > 0.f && c->v_scale[g] < 3.0e38f))
        return fail(FLINT_ERR_INVALID_ARG, "%s: E4M3 scales must be finite and > 0", who);
  if (!aligned16(c->k) || !aligned16(c->v))
    return fail(FLINT_ERR_INVALID_ARG, "%s: cache k/v must be 16-byte aligned", who);
  switch (c->layout) {
    case FLINT_KV_CONTIGUOUS:
    case FLINT_KV_RING: {
      if (c->capacity < 1 || c->capacity > FLINT_MAX_CONTEXT)
        return fail(FLINT_ERR_INVALID_ARG, "%s: capacity %d out of range", who, c->capacity);
      if (c->layout == FLINT_KV_RING && c->capacity != kWindow)
        return fail(FLINT_ERR_UNSUPPORTED, "%s: a ring cache must have %d slots", who, kWindow);
      const int64_t dense = static_cast<int64_t>(c->capacity) * kKvHeads * kDim;
      const int64_t mult = c->dtype == FLINT_KV_FP8_E4M3 ? 16 : 8;  // 16-byte TMA strides
      if (c->req_stride != 0 && (c->req_stride < dense || c->req_stride % mult != 0))
        return fail(FLINT_ERR_INVALID_ARG, "%s: req_stride %lld must be 0 or a multiple of %lld >= %lld",
                    who, (long long)c->req_stride, (long long)mult, (long long)dense);
      (void)B;
      return FLINT_OK;
    }
    case FLINT_KV_PAGED:
      if (!c->block_table) return fail(FLINT_ERR_INVALID_ARG, "%s: block_table is NULL", who);
      if (c->block_size != kBlock)
        return fail(FLINT_ERR_UNSUPPORTED, "%s: block_size must be %d", who, kBlock);
      if (c->max_blocks_per_req < 1 || c->num_blocks < 1)
        return fail(FLINT_ERR_INVALID_ARG, "%s: max_blocks_per_req and num_blocks must be >= 1", who);
      return FLINT_OK;
    default:
      return fail(FLINT_ERR_INVALID_ARG, "%s: unknown cache layout %d", who, c->layout);
  }
}

// Attended range of one request in storage coordinates, plus its tiles.
struct Range {
  int lo, hi, tile_base, tiles;
};

Range attended_range(const flint_kv_cache& c, int L, int window) {
  const int T = c.dtype == FLINT_KV_FP8_E4M3 ? kTileFp8 : kTile;  // tokens per tile
  Range r;
  if (c.layout == FLINT_KV_RING) {
    r.lo = 0;
    r.hi = std::min(L, c.capacity);
    r.tile_base = 0;
  } else {
    r.lo = window > 0 ? std::max(0, L - window) : 0;
    r.hi = L;
    // paged tiles must not straddle a block: start them on a multiple of T
    r.tile_base = c.layout == FLINT_KV_PAGED ? (r.lo / T) * T : r.lo;
  }
  r.tiles = (r.hi - r.tile_base + T - 1) / T;
  return r;
}

flint_status check_len(const flint_kv_cache& c, int L, int window, const char* who, int idx) {
  if (L < 1 || L > FLINT_MAX_CONTEXT)
    return fail(FLINT_ERR_INVALID_ARG, "%s: length %d of item %d outside [1, %d]", who, L, idx,
                FLINT_MAX_CONTEXT);
  if (c.layout == FLINT_KV_CONTIGUOUS && L > c.capacity)
    return fail(FLINT_ERR_INVALID_ARG, "%s: length %d of item %d exceeds capacity %d", who, L, idx,
                c.capacity);
  if (c.layout == FLINT_KV_RING && window != kWindow)
    return fail(FLINT_ERR_UNSUPPORTED, "%s: a ring cache needs window %d", who, kWindow);
  if (c.layout == FLINT_KV_PAGED &&
      static_cast<int64_t>(L) > static_cast<int64_t>(c.max_blocks_per_req) * kBlock)
    return fail(FLINT_ERR_INVALID_ARG, "%s: length %d of item %d exceeds the block table (%d blocks)",
                who, L, idx, c.max_blocks_per_req);
  return FLINT_OK;
}

constexpr size_t kPartialBytes = kPartialFloats * sizeof(float);

// Fill plan fields of P from the problems' tile counts; returns the grid.  The
// workspace must hold the static plan (at most G + n_problems - 1 items); the
// run-time queue gets what the rest of it (and kMaxItems) allows.
flint_status plan(DecodeParams& P, const int* tiles, int n_problems, int num_ctas, size_t ws_bytes,
                  const char* who, int* grid) {
  int sms = num_ctas;
  if (sms == 0 && device_num_sms(&sms) != 0)
    return fail(FLINT_ERR_CUDA, "cannot query the SM count of the current device");
  // One CTA fits an SM, and a launch whose merging CTAs wait for the others needs all of
  // them resident: never more CTAs than the device has SMs.
  int dev_sms = 0;
  if (num_ctas > 0 && device_num_sms(&dev_sms) == 0) sms = std::min(sms, dev_sms);
  sms = std::min(sms, kMaxCtas);
  int32_t seg_tiles[kMaxSegs];
  int64_t total = 0;
  for (int p = 0; p < n_problems; ++p) {
    seg_tiles[p] = tiles[p];
    total += tiles[p];
  }
  const int n_segs = n_problems;
  // at least two tiles of work per CTA, never more CTAs than the device's SMs
  const int G = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(sms, (total + 1) / 2)));
  const size_t need = kCounterBytes + static_cast<size_t>(std::min(kMaxItems, G + n_problems)) * kPartialBytes;
  if (ws_bytes < need)
    return fail(FLINT_ERR_WORKSPACE, "%s: workspace of %zu bytes is below the %zu needed", who, ws_bytes, need);
  const int cap = static_cast<int>(std::min<size_t>(kMaxItems, (ws_bytes - kCounterBytes) / kPartialBytes));
  int32_t seg[kMaxItems], t0[kMaxItems], t1[kMaxItems], order[kMaxItems], cb[kMaxCtas + 1];
  const int n = flint_plan_split(seg_tiles, n_segs, G, kItemCost, cap, seg, t0, t1, order, cb);
  if (n < 0) return fail(FLINT_ERR_UNSUPPORTED, "%s: split plan does not fit one launch", who);
  bool queued[kMaxSegs] = {};
  for (int i = 0; i < n; ++i) {
    P.items[i].seg = static_cast<int16_t>(seg[i]);
    P.items[i].t0 = static_cast<int16_t>(t0[i]);
    P.items[i].t1 = static_cast<int16_t>(t1[i]);
    P.items[i].pad = 0;
    P.order[i] = static_cast<int16_t>(order[i]);
  }
  P.n_items = n;
  P.queue_begin = cb[G];
  P.n_queue = n - cb[G];
  for (int q = P.queue_begin; q < n; ++q) queued[seg[order[q]]] = true;
  int last = 0;  // with no queue, CTAs past the last one with work are not launched
  for (int c = 0; c < G; ++c) {
    P.cta_item_begin[c] = static_cast<int16_t>(cb[c]);
    if (cb[c + 1] > cb[c]) last = c + 1;
  }
  P.cta_item_begin[G] = static_cast<int16_t>(cb[G]);
  for (int s = 0, i = 0; s <= n_segs; ++s) {
    while (i < n && seg[i] < s) ++i;
    P.seg_item_begin[s] = static_cast<int16_t>(i);
  }
  // Problems with queued chunks, or split more widely than kInlineMergeMax,
  // are merged at the launch's end by the whole grid (after a grid barrier,
  // or on ready flags, see below): their last items finish near the end of
  // the launch, where one CTA merging alone would be the tail.
  P.n_deferred = 0;
  P.n_wide = 0;
  // When a CTA per unit covers every unit of every deferred problem at once
  // (a lone problem on a short context), every problem is merged that way:
  // each warp then folds a ninth of the partials.
  int n_def = 0;
  for (int s = 0; s < n_segs; ++s)
    n_def += (queued[s] || P.seg_item_begin[s + 1] - P.seg_item_begin[s] > kInlineMergeMax) ? 1 : 0;
  const bool one_round = n_def * kKvHeads * 8 <= G;
  for (int wide = 1; wide >= 0; --wide) {
    for (int s = 0; s < n_segs; ++s) {
      const int items = P.seg_item_begin[s + 1] - P.seg_item_begin[s];
      const bool deferred = queued[s] || items > kInlineMergeMax;
      P.prob[s].deferred = deferred ? 1 : 0;
      if (deferred && (items > kWideMergeItems || one_round) == (wide == 1)) P.deferred[P.n_deferred++] = static_cast<int16_t>(s);
    }
    if (wide) P.n_wide = P.n_deferred;
  }
  for (int w = 0; w < kMaxItems / 32; ++w) P.raised[w] = 0;
  for (int i = 0; i < n; ++i)
    if (P.prob[seg[i]].deferred) P.raised[i / 32] |= 1u << (i % 32);
  P.grid_merge = (P.n_deferred > 0 || P.n_queue > 0) ? 1 : 0;
  // Ready flags where a problem is split over very many items (a lone long
  // context over every SM), the grid barrier otherwise.
  P.merge_flags = 0;
  for (int s = 0; s < n_segs; ++s)
    if (P.seg_item_begin[s + 1] - P.seg_item_begin[s] > kWideMergeItems) P.merge_flags = P.grid_merge;
  P.ws_items = cap;
  *grid = P.n_queue > 0 ? G : last;
  return FLINT_OK;
}

// E4M3 scales of the cache behind map pair `pair` (read by the kernel as
// kv_scales[map_k / 2]); zero for a bf16 cache.
void set_scales(DecodeParams& P, int pair, const flint_kv_cache& c) {
  for (int g = 0; g < kKvHeads; ++g) {
    const bool fp8 = c.dtype == FLINT_KV_FP8_E4M3;
    P.kv_scales[pair][g] = fp8 ? c.k_scale[g] : 0.f;
    P.kv_scales[pair][4 + g] = fp8 ? c.v_scale[g] : 0.f;
  }
}

void set_prep_fp8(PrepParams& p, const flint_kv_cache& c) {
  p.fp8 = c.dtype == FLINT_KV_FP8_E4M3 ? 1 : 0;
  for (int g = 0; g < kKvHeads; ++g) {
    p.k_scale[g] = p.fp8 ? c.k_scale[g] : 0.f;
    p.v_scale[g] = p.fp8 ? c.v_scale[g] : 0.f;
  }
}

flint_status launch_result(cudaError_t e, const char* who) {
  if (e != cudaSuccess) return fail(FLINT_ERR_CUDA, "%s: launch failed: %s", who, cudaGetErrorString(e));
  return ok();
}

}  // namespace

namespace {

flint_status run_stack(const flint_layer* layers, int32_t n_layers, int32_t pos, float eps, double theta,
                       float* out, void* workspace, size_t ws_bytes, int32_t num_ctas, int32_t* dev_err,
                       void* stream, int pdl, const char* who) {
  if (!layers || !out || !workspace) return fail(FLINT_ERR_INVALID_ARG, "%s: NULL pointer argument", who);
  if (n_layers < 1 || n_layers > FLINT_MAX_LAYERS)
    return fail(FLINT_ERR_INVALID_ARG, "%s: n_layers=%d outside [1, %d]", who, n_layers, FLINT_MAX_LAYERS);
  if (pos < 0 || pos >= FLINT_MAX_CONTEXT) return fail(FLINT_ERR_INVALID_ARG, "%s: pos=%d outside [0, %d)", who, pos, FLINT_MAX_CONTEXT);
  if (!(eps >= 0.f) || !(theta > 0.0)) return fail(FLINT_ERR_INVALID_ARG, "%s: eps must be >= 0, theta > 0", who);
  if (num_ctas < 0 || num_ctas > kMaxCtas) return fail(FLINT_ERR_INVALID_ARG, "%s: num_ctas %d outside [0, %d]", who, num_ctas, kMaxCtas);
  if (!aligned16(out) || !aligned16(workspace)) return fail(FLINT_ERR_INVALID_ARG, "%s: out/workspace must be 16-byte aligned", who);
  const int L = pos + 1;
  int tiles[kMaxProblems];
  static thread_local DecodeParams P;
  memset(&P, 0, sizeof P);
  for (int i = 0; i < n_layers; ++i) {
    const flint_layer& ly = layers[i];
    if (!ly.q_raw || !ly.k_raw || !ly.v_raw || !ly.w_q || !ly.w_k || !ly.sinks)
      return fail(FLINT_ERR_INVALID_ARG, "%s: layer %d has a NULL pointer", who, i);
    const void* ptrs[] = {ly.q_raw, ly.k_raw, ly.v_raw, ly.w_q, ly.w_k};
    for (const void* p : ptrs)
      if (!aligned16(p)) return fail(FLINT_ERR_INVALID_ARG, "%s: layer %d pointers must be 16-byte aligned", who, i);
    if (ly.window != 0 && ly.window != kWindow)
      return fail(FLINT_ERR_UNSUPPORTED, "%s: layer %d window must be 0 or %d", who, i, kWindow);
    if (ly.rope != 0 && ly.rope != 1) return fail(FLINT_ERR_INVALID_ARG, "%s: layer %d rope must be 0 or 1", who, i);
    flint_status s = check_cache(&ly.cache, 1, who);
    if (s != FLINT_OK) return s;
    s = check_len(ly.cache, L, ly.window, who, i);
    if (s != FLINT_OK) return s;
    const Range r = attended_range(ly.cache, L, ly.window);
    Problem& pb = P.prob[i];
    pb.q = ly.q_raw;
    pb.k_raw = ly.k_raw;
    pb.v_raw = ly.v_raw;
    pb.w_q = ly.w_q;
    pb.w_k = ly.w_k;
    pb.sinks = ly.sinks;
    pb.out = out + static_cast<size_t>(i) * kHeads * kDim;
    pb.k_rows = static_cast<uint16_t*>(ly.cache.k);
    pb.v_rows = static_cast<uint16_t*>(ly.cache.v);
    pb.table = ly.cache.layout == FLINT_KV_PAGED ? ly.cache.block_table : nullptr;
    pb.lo = r.lo;
    pb.hi = r.hi;
    pb.tile_base = r.tile_base;
    pb.pos = pos;
    pb.append_tok = ly.cache.layout == FLINT_KV_RING ? pos % ly.cache.capacity : pos;
    pb.num_blocks = ly.cache.num_blocks;
    pb.ext2 = ly.cache.layout == FLINT_KV_PAGED ? kBlock : ly.cache.capacity;
    pb.ext3 = ly.cache.layout == FLINT_KV_PAGED ? ly.cache.num_blocks : 1;
    pb.table_len = ly.cache.layout == FLINT_KV_PAGED ? ly.cache.max_blocks_per_req : 0;
    pb.map_k = static_cast<int16_t>(2 * i);
    pb.map_v = static_cast<int16_t>(2 * i + 1);
    pb.req = 0;
    pb.layout = static_cast<int8_t>(ly.cache.layout);
    pb.q_fp32 = 0;
    pb.rope = static_cast<int8_t>(ly.rope);
    pb.fp8 = static_cast<int8_t>(ly.cache.dtype == FLINT_KV_FP8_E4M3);
    set_scales(P, i, ly.cache);
    tiles[i] = r.tiles;
    s = encode_cache_map(&P.maps[2 * i], ly.cache.k, ly.cache, 1);
    if (s != FLINT_OK) return s;
    s = encode_cache_map(&P.maps[2 * i + 1], ly.cache.v, ly.cache, 1);
    if (s != FLINT_OK) return s;
  }
  int grid = 0;
  flint_status s = plan(P, tiles, n_layers, num_ctas, ws_bytes, who, &grid);
  if (s != FLINT_OK) return s;
  P.smem_bytes = static_cast<int32_t>(decode_smem_bytes());
  P.counters = static_cast<int32_t*>(workspace);
  P.partials = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kCounterBytes);
  P.dev_err = dev_err;
  P.n_problems = n_layers;
  P.prep = 1;
  P.pdl = pdl;
  // A launch that depends on the previous one (layer-serial stack) keeps the
  // grid-barrier merge: there the ready-flag mode measured 3.3 us slower per
  // full layer (1,079 -> 1,125 us for 49 dependent layers).
  if (pdl) P.merge_flags = 0;
  P.eps = eps;
  // RoPE angles of the new token, pos * theta^(-2i/128) for i < 64, in double
  // on the host (one position for every layer of the call)
  for (int i = 0; i < kDim / 2; ++i) {
    const double a = static_cast<double>(pos) * std::pow(theta, -2.0 * i / kDim);
    P.rope_cs[i] = make_float2(static_cast<float>(std::cos(a)), static_cast<float>(std::sin(a)));
  }
  return launch_result(launch_decode(P, grid, static_cast<cudaStream_t>(stream)), who);
}

}  // namespace

namespace flint {

size_t workspace_min_bytes(int n_problems, int num_ctas) {
  if (n_problems < 1 || n_problems > kMaxProblems || num_ctas < 0 || num_ctas > kMaxCtas) return 0;
  // the CTAs plan() launches: num_ctas (0: one per SM), never more than the
  // device's SMs (kMaxCtas if the count cannot be read)
  int sms = kMaxCtas;
  if (device_num_sms(&sms) != 0) sms = kMaxCtas;
  const int g = std::min(num_ctas == 0 ? sms : std::min(num_ctas, sms), kMaxCtas);
  return kCounterBytes + static_cast<size_t>(std::min(kMaxItems, g + n_problems)) * kPartialBytes;
}

void* current_context() {
  typedef CUresult (*GetCtxFn)(CUcontext*);
  static GetCtxFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<GetCtxFn>(p);
  });
  CUcontext ctx = nullptr;
  if (!fn || fn(&ctx) != CUDA_SUCCESS) return nullptr;
  return ctx;
}

cudaError_t configure_once(ContextSet& done, const void* kernel, int bytes) {
  void* ctx = current_context();
  std::lock_guard<std::mutex> lock(done.mu);
  if (ctx && std::find(done.ctxs.begin(), done.ctxs.end(), ctx) != done.ctxs.end()) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  // with no context yet the call above made one; the next launch records it
  if (ctx) done.ctxs.push_back(ctx);
  return cudaSuccess;
}

flint_status record_error(flint_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

}  // namespace flint

extern "C" {

const char* flint_status_string(flint_status s) {
  switch (s) {
    case FLINT_OK: return "ok";
    case FLINT_ERR_INVALID_ARG: return "invalid argument";
    case FLINT_ERR_UNSUPPORTED: return "unsupported";
    case FLINT_ERR_WORKSPACE: return "workspace too small";
    case FLINT_ERR_CUDA: return "CUDA error";
    case FLINT_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

const char* flint_last_error(void) { return g_last_error.c_str(); }

uint64_t flint_kv_bytes(int64_t ctx_len, int32_t n_full, int32_t n_window, int32_t window,
                        int32_t elem_bytes) {
  if (ctx_len < 0 || n_full < 0 || n_window < 0 || window < 0 || elem_bytes < 0) return 0;
  const uint64_t per_tok = 2ull * kKvHeads * kDim * static_cast<uint64_t>(elem_bytes);
  const uint64_t kept = static_cast<uint64_t>(std::min<int64_t>(ctx_len, window));
  return per_tok * (static_cast<uint64_t>(n_full) * static_cast<uint64_t>(ctx_len) +
                    static_cast<uint64_t>(n_window) * kept);
}

flint_status flint_qk_norm_rope(const uint16_t* q_raw, const uint16_t* k_raw, const uint16_t* v_raw,
                                const uint16_t* w_q, const uint16_t* w_k, const int32_t* pos,
                                int32_t B, float eps, double theta, int32_t apply_rope,
                                float* q_out, uint16_t* k_out, const flint_kv_cache* cache,
                                int32_t* dev_err, void* stream) {
  FLINT_NVTX_RANGE("flint_qk_norm_rope");
  const char* who = "flint_qk_norm_rope";
  if (!q_raw || !k_raw || !w_q || !w_k || !pos)
    return fail(FLINT_ERR_INVALID_ARG, "%s: NULL input pointer", who);
  if (B < 1 || B > FLINT_MAX_BATCH) return fail(FLINT_ERR_INVALID_ARG, "%s: B=%d outside [1, %d]", who, B, FLINT_MAX_BATCH);
  if (apply_rope != 0 && apply_rope != 1) return fail(FLINT_ERR_INVALID_ARG, "%s: apply_rope must be 0 or 1", who);
  if (!(eps >= 0.f) || !(theta > 0.0)) return fail(FLINT_ERR_INVALID_ARG, "%s: eps must be >= 0, theta > 0", who);
  if (!q_out && !k_out && !cache) return fail(FLINT_ERR_INVALID_ARG, "%s: no output requested", who);
  const void* ptrs[] = {q_raw, k_raw, w_q, w_k, q_out, k_out, v_raw};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(FLINT_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", who);
  PrepParams p;
  memset(&p, 0, sizeof p);
  p.q_raw = q_raw;
  p.k_raw = k_raw;
  p.v_raw = v_raw;
  p.w_q = w_q;
  p.w_k = w_k;
  p.q_out = q_out;
  p.k_out = k_out;
  p.eps = eps;
  p.theta = theta;
  p.apply_rope = apply_rope;
  p.do_norm = 1;
  p.dev_err = dev_err;
  for (int b = 0; b < B; ++b) {
    if (pos[b] < 0 || pos[b] >= FLINT_MAX_CONTEXT)
      return fail(FLINT_ERR_INVALID_ARG, "%s: pos[%d]=%d outside [0, %d)", who, b, pos[b], FLINT_MAX_CONTEXT);
    p.pos[b] = pos[b];
  }
  if (cache) {
    if (!v_raw) return fail(FLINT_ERR_INVALID_ARG, "%s: appending needs v_raw", who);
    flint_status s = check_cache(cache, B, who);
    if (s != FLINT_OK) return s;
    for (int b = 0; b < B; ++b) {
      const flint_kv_cache& c = *cache;
      if (c.layout == FLINT_KV_CONTIGUOUS && pos[b] >= c.capacity)
        return fail(FLINT_ERR_INVALID_ARG, "%s: pos[%d]=%d outside the cache capacity %d", who, b, pos[b], c.capacity);
      if (c.layout == FLINT_KV_PAGED && pos[b] / kBlock >= c.max_blocks_per_req)
        return fail(FLINT_ERR_INVALID_ARG, "%s: pos[%d]=%d outside the block table", who, b, pos[b]);
    }
    p.k_rows = static_cast<uint16_t*>(cache->k);
    p.v_rows = static_cast<uint16_t*>(cache->v);
    p.table = cache->block_table;
    p.layout = cache->layout;
    p.capacity = cache->capacity;
    p.req_stride = cache->req_stride ? cache->req_stride
                                     : static_cast<int64_t>(cache->capacity) * kKvHeads * kDim;
    p.max_blocks = cache->max_blocks_per_req;
    p.num_blocks = cache->num_blocks;
    set_prep_fp8(p, *cache);
  }
  return launch_result(launch_prep(p, B, static_cast<cudaStream_t>(stream)), who);
}

flint_status flint_kv_append(const uint16_t* k, const uint16_t* v, const int32_t* pos, int32_t B,
                             const flint_kv_cache* cache, int32_t* dev_err, void* stream) {
  FLINT_NVTX_RANGE("flint_kv_append");
  const char* who = "flint_kv_append";
  if (!k || !v || !pos) return fail(FLINT_ERR_INVALID_ARG, "%s: NULL input pointer", who);
  if (!aligned16(k) || !aligned16(v)) return fail(FLINT_ERR_INVALID_ARG, "%s: k/v must be 16-byte aligned", who);
  if (B < 1 || B > FLINT_MAX_BATCH) return fail(FLINT_ERR_INVALID_ARG, "%s: B=%d outside [1, %d]", who, B, FLINT_MAX_BATCH);
  flint_status s = check_cache(cache, B, who);
  if (s != FLINT_OK) return s;
  PrepParams p;
  memset(&p, 0, sizeof p);
  p.k_raw = k;
  p.v_raw = v;
  p.dev_err = dev_err;
  p.do_norm = 0;
  p.apply_rope = 0;
  for (int b = 0; b < B; ++b) {
    if (pos[b] < 0 || pos[b] >= FLINT_MAX_CONTEXT)
      return fail(FLINT_ERR_INVALID_ARG, "%s: pos[%d]=%d outside [0, %d)", who, b, pos[b], FLINT_MAX_CONTEXT);
    if (cache->layout == FLINT_KV_CONTIGUOUS && pos[b] >= cache->capacity)
      return fail(FLINT_ERR_INVALID_ARG, "%s: pos[%d]=%d outside the cache capacity %d", who, b, pos[b], cache->capacity);
    if (cache->layout == FLINT_KV_PAGED && pos[b] / kBlock >= cache->max_blocks_per_req)
      return fail(FLINT_ERR_INVALID_ARG, "%s: pos[%d]=%d outside the block table", who, b, pos[b]);
    p.pos[b] = pos[b];
  }
  p.k_rows = static_cast<uint16_t*>(cache->k);
  p.v_rows = static_cast<uint16_t*>(cache->v);
  p.table = cache->block_table;
  p.layout = cache->layout;
  p.capacity = cache->capacity;
  p.req_stride = cache->req_stride ? cache->req_stride
                                   : static_cast<int64_t>(cache->capacity) * kKvHeads * kDim;
  p.max_blocks = cache->max_blocks_per_req;
  p.num_blocks = cache->num_blocks;
  set_prep_fp8(p, *cache);
  return launch_result(launch_prep(p, B, static_cast<cudaStream_t>(stream)), who);
}

flint_status flint_prefill_qk_norm_rope(const uint16_t* q_raw, const uint16_t* k_raw,
                                        const uint16_t* v_raw, const uint16_t* w_q,
                                        const uint16_t* w_k, int32_t T, float eps,
                                        double theta, int32_t apply_rope, uint16_t* q_out,
                                        uint16_t* k_out, uint16_t* v_out,
                                        const flint_kv_cache* cache, int32_t* dev_err,
                                        void* stream) {
  FLINT_NVTX_RANGE("flint_prefill_qk_norm_rope");
  const char* who = "flint_prefill_qk_norm_rope";
  if (!q_raw || !k_raw || !w_q || !w_k) return fail(FLINT_ERR_INVALID_ARG, "%s: NULL input pointer", who);
  if (T < 1 || T > FLINT_MAX_CONTEXT)
    return fail(FLINT_ERR_INVALID_ARG, "%s: T=%d outside [1, %d]", who, T, FLINT_MAX_CONTEXT);
  if (apply_rope != 0 && apply_rope != 1) return fail(FLINT_ERR_INVALID_ARG, "%s: apply_rope must be 0 or 1", who);
  if (!(eps >= 0.f) || !(theta > 0.0)) return fail(FLINT_ERR_INVALID_ARG, "%s: eps must be >= 0, theta > 0", who);
  if (!q_out && !k_out && !v_out && !cache) return fail(FLINT_ERR_INVALID_ARG, "%s: no output requested", who);
  if (v_out && !v_raw) return fail(FLINT_ERR_INVALID_ARG, "%s: v_out needs v_raw", who);
  const void* ptrs[] = {q_raw, k_raw, w_q, w_k, q_out, k_out, v_out, v_raw};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(FLINT_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", who);
  PrepParams p;
  memset(&p, 0, sizeof p);
  p.q_raw = q_raw;
  p.k_raw = k_raw;
  p.v_raw = v_raw;
  p.w_q = w_q;
  p.w_k = w_k;
  p.q_out_bf16 = q_out;
  p.v_out_f16 = v_out;
  p.k_out = k_out;
  p.eps = eps;
  p.theta = theta;
  p.apply_rope = apply_rope;
  p.do_norm = 1;
  p.dev_err = dev_err;
  p.prefill = 1;
  p.n_tokens = T;
  if (cache) {
    if (!v_raw) return fail(FLINT_ERR_INVALID_ARG, "%s: writing the cache needs v_raw", who);
    flint_status s = check_cache(cache, 1, who);
    if (s != FLINT_OK) return s;
    const flint_kv_cache& c = *cache;
    if (c.layout == FLINT_KV_CONTIGUOUS && T > c.capacity)
      return fail(FLINT_ERR_INVALID_ARG, "%s: T=%d exceeds the cache capacity %d", who, T, c.capacity);
    if (c.layout == FLINT_KV_PAGED && static_cast<int64_t>(T) > static_cast<int64_t>(c.max_blocks_per_req) * kBlock)
      return fail(FLINT_ERR_INVALID_ARG, "%s: T=%d exceeds the block table (%d blocks)", who, T, c.max_blocks_per_req);
    p.k_rows = static_cast<uint16_t*>(c.k);
    p.v_rows = static_cast<uint16_t*>(c.v);
    p.table = c.block_table;
    p.layout = c.layout;
    p.capacity = c.capacity;
    p.req_stride = c.req_stride ? c.req_stride : static_cast<int64_t>(c.capacity) * kKvHeads * kDim;
    p.max_blocks = c.max_blocks_per_req;
    p.num_blocks = c.num_blocks;
    set_prep_fp8(p, c);
  }
  int sms = 0;
  if (device_num_sms(&sms) != 0) return fail(FLINT_ERR_CUDA, "%s: cannot read the device's SM count", who);
  return launch_result(launch_prefill_prep(p, prefill_prep_grid(T, sms), static_cast<cudaStream_t>(stream)), who);
}

flint_status flint_prefill_attn(const uint16_t* q, const uint16_t* k, const uint16_t* v, int32_t T,
                                const float* sinks, int32_t window, float* out, int32_t* dev_err,
                                void* stream) {
  FLINT_NVTX_RANGE("flint_prefill_attn");
  const char* who = "flint_prefill_attn";
  if (!q || !k || !v || !sinks || !out) return fail(FLINT_ERR_INVALID_ARG, "%s: NULL pointer", who);
  const void* ptrs[] = {q, k, v, sinks, out};
  for (const void* p : ptrs)
    if (!aligned16(p)) return fail(FLINT_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", who);
  if (T < 1 || T > FLINT_MAX_CONTEXT)
    return fail(FLINT_ERR_INVALID_ARG, "%s: T=%d outside [1, %d]", who, T, FLINT_MAX_CONTEXT);
  if (window != 0 && window != kWindow)
    return fail(FLINT_ERR_UNSUPPORTED, "%s: window must be 0 or %d", who, kWindow);
  PrefillParams p;
  memset(&p, 0, sizeof p);
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(FLINT_ERR_CUDA, "%s: cuTensorMapEncodeTiled is not available from the driver", who);
  // [128 dims][heads][T tokens][1] bf16, 128-byte swizzle, boxes of 64 dims
  auto encode = [&](CUtensorMap* map, const void* base, int heads, int box_heads, int box_tokens,
                    CUtensorMapDataType dtype) {
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(kDim), static_cast<cuuint64_t>(heads),
                                static_cast<cuuint64_t>(T), 1};
    const cuuint64_t strides[3] = {kDim * 2ull, static_cast<cuuint64_t>(heads) * kDim * 2ull,
                                   static_cast<cuuint64_t>(T) * heads * kDim * 2ull};
    const cuuint32_t box[4] = {64, static_cast<cuuint32_t>(box_heads), static_cast<cuuint32_t>(box_tokens), 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(map, dtype, 4, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  };
  if (encode(&p.q_map, q, kHeads, kGroup, 16, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) != CUDA_SUCCESS ||
      encode(&p.k_map, k, kKvHeads, 1, 128, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) != CUDA_SUCCESS ||
      encode(&p.v_map, v, kKvHeads, 1, 128, CU_TENSOR_MAP_DATA_TYPE_FLOAT16) != CUDA_SUCCESS)
    return fail(FLINT_ERR_CUDA, "%s: cuTensorMapEncodeTiled failed", who);
  p.sinks = sinks;
  p.out = out;
  p.dev_err = dev_err;
  p.T = T;
  p.window = window;
  int sms = 0;
  if (device_num_sms(&sms) != 0) return fail(FLINT_ERR_CUDA, "%s: cannot read the device's SM count", who);
  return launch_result(launch_prefill(p, sms, static_cast<cudaStream_t>(stream)), who);
}

size_t flint_attn_workspace_bytes(int32_t n_problems, int32_t num_ctas) {
  if (n_problems < 1 || n_problems > kMaxProblems || num_ctas < 0 || num_ctas > kMaxCtas) return 0;
  return kCounterBytes + static_cast<size_t>(kMaxItems) * kPartialBytes;
}

static flint_status decode_impl(const void* q, int32_t q_is_fp32, const flint_kv_cache* cache,
                                const int32_t* seq_lens, int32_t B, const float* sinks, int32_t window,
                                float* out, void* workspace, size_t ws_bytes, int32_t num_ctas,
                                int32_t* dev_err, void* stream, bool partial, const char* who) {
  if (!q || !seq_lens || (!sinks && !partial) || !out || !workspace)
    return fail(FLINT_ERR_INVALID_ARG, "%s: NULL pointer argument", who);
  if (B < 1 || B > FLINT_MAX_BATCH) return fail(FLINT_ERR_INVALID_ARG, "%s: B=%d outside [1, %d]", who, B, FLINT_MAX_BATCH);
  if (q_is_fp32 != 0 && q_is_fp32 != 1) return fail(FLINT_ERR_INVALID_ARG, "%s: q_is_fp32 must be 0 or 1", who);
  if (window != 0 && window != kWindow) return fail(FLINT_ERR_UNSUPPORTED, "%s: window must be 0 or %d", who, kWindow);
  if (num_ctas < 0 || num_ctas > kMaxCtas) return fail(FLINT_ERR_INVALID_ARG, "%s: num_ctas %d outside [0, %d]", who, num_ctas, kMaxCtas);
  if (!aligned16(q) || !aligned16(out) || !aligned16(workspace) || (reinterpret_cast<uintptr_t>(sinks) & 3u))
    return fail(FLINT_ERR_INVALID_ARG, "%s: q/out/workspace must be 16-byte aligned", who);
  flint_status s = check_cache(cache, B, who);
  if (s != FLINT_OK) return s;
  int tiles[kMaxProblems];
  static thread_local DecodeParams P;
  memset(&P, 0, sizeof P);
  for (int b = 0; b < B; ++b) {
    s = check_len(*cache, seq_lens[b], window, who, b);
    if (s != FLINT_OK) return s;
    const Range r = attended_range(*cache, seq_lens[b], window);
    Problem& pb = P.prob[b];
    pb.q = static_cast<const uint8_t*>(q) + static_cast<size_t>(b) * kHeads * kDim * (q_is_fp32 ? 4 : 2);
    pb.sinks = partial ? nullptr : sinks;
    pb.out = out + static_cast<size_t>(b) * (partial ? kCpPartialFloats : kHeads * kDim);
    pb.partial = static_cast<int8_t>(partial);
    pb.table = cache->layout == FLINT_KV_PAGED
                   ? cache->block_table + static_cast<size_t>(b) * cache->max_blocks_per_req
                   : nullptr;
    pb.lo = r.lo;
    pb.hi = r.hi;
    pb.tile_base = r.tile_base;
    pb.append_tok = -1;
    pb.pos = seq_lens[b] - 1;
    pb.num_blocks = cache->num_blocks;
    pb.ext2 = cache->layout == FLINT_KV_PAGED ? kBlock : cache->capacity;
    pb.ext3 = cache->layout == FLINT_KV_PAGED ? cache->num_blocks : B;
    pb.table_len = cache->layout == FLINT_KV_PAGED ? cache->max_blocks_per_req : 0;
    pb.map_k = 0;
    pb.map_v = 1;
    pb.req = static_cast<int16_t>(cache->layout == FLINT_KV_PAGED ? 0 : b);
    pb.layout = static_cast<int8_t>(cache->layout);
    pb.q_fp32 = static_cast<int8_t>(q_is_fp32);
    pb.fp8 = static_cast<int8_t>(cache->dtype == FLINT_KV_FP8_E4M3);
    tiles[b] = r.tiles;
  }
  int grid = 0;
  s = plan(P, tiles, B, num_ctas, ws_bytes, who, &grid);
  if (s != FLINT_OK) return s;
  set_scales(P, 0, *cache);
  s = encode_cache_map(&P.maps[0], cache->k, *cache, B);
  if (s != FLINT_OK) return s;
  s = encode_cache_map(&P.maps[1], cache->v, *cache, B);
  if (s != FLINT_OK) return s;
  P.smem_bytes = static_cast<int32_t>(decode_smem_bytes());
  P.counters = static_cast<int32_t*>(workspace);
  P.partials = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kCounterBytes);
  P.dev_err = dev_err;
  P.n_problems = B;
  P.prep = 0;
  P.eps = 0.f;
  return launch_result(launch_decode(P, grid, static_cast<cudaStream_t>(stream)), who);
}

flint_status flint_attn_decode(const void* q, int32_t q_is_fp32, const flint_kv_cache* cache,
                               const int32_t* seq_lens, int32_t B, const float* sinks,
                               int32_t window, float* out, void* workspace, size_t ws_bytes,
                               int32_t num_ctas, int32_t* dev_err, void* stream) {
  FLINT_NVTX_RANGE("flint_attn_decode");
  return decode_impl(q, q_is_fp32, cache, seq_lens, B, sinks, window, out, workspace, ws_bytes, num_ctas,
                     dev_err, stream, false, "flint_attn_decode");
}

flint_status flint_attn_decode_partial(const void* q, int32_t q_is_fp32, const flint_kv_cache* cache,
                                       const int32_t* seq_lens, int32_t B, float* partials,
                                       void* workspace, size_t ws_bytes, int32_t num_ctas,
                                       int32_t* dev_err, void* stream) {
  FLINT_NVTX_RANGE("flint_attn_decode_partial");
  return decode_impl(q, q_is_fp32, cache, seq_lens, B, nullptr, 0, partials, workspace, ws_bytes, num_ctas,
                     dev_err, stream, true, "flint_attn_decode_partial");
}

flint_status flint_merge_partials(const float* partials, int32_t n_parts, int32_t B, const float* sinks,
                                  float* out, void* stream) {
  FLINT_NVTX_RANGE("flint_merge_partials");
  const char* who = "flint_merge_partials";
  if (!partials || !sinks || !out) return fail(FLINT_ERR_INVALID_ARG, "%s: NULL pointer argument", who);
  if (n_parts < 1 || n_parts > FLINT_MAX_CP_PARTS)
    return fail(FLINT_ERR_INVALID_ARG, "%s: n_parts=%d outside [1, %d]", who, n_parts, FLINT_MAX_CP_PARTS);
  if (B < 1 || B > FLINT_MAX_BATCH) return fail(FLINT_ERR_INVALID_ARG, "%s: B=%d outside [1, %d]", who, B, FLINT_MAX_BATCH);
  if (!aligned16(partials) || !aligned16(out) || (reinterpret_cast<uintptr_t>(sinks) & 3u))
    return fail(FLINT_ERR_INVALID_ARG, "%s: partials/out must be 16-byte aligned", who);
  return launch_result(launch_merge_partials(partials, n_parts, B, sinks, out, static_cast<cudaStream_t>(stream)),
                       who);
}

flint_status flint_attn_stack(const flint_layer* layers, int32_t n_layers, int32_t pos, float eps,
                              double theta, float* out, void* workspace, size_t ws_bytes,
                              int32_t num_ctas, int32_t* dev_err, void* stream) {
  FLINT_NVTX_RANGE("flint_attn_stack");
  return run_stack(layers, n_layers, pos, eps, theta, out, workspace, ws_bytes, num_ctas, dev_err, stream, 0,
                   "flint_attn_stack");
}

flint_status flint_attn_layers_serial(const flint_layer* layers, int32_t n_layers, int32_t pos, float eps,
                                      double theta, float* out, void* workspace, size_t ws_bytes,
                                      int32_t num_ctas, int32_t* dev_err, void* stream) {
  FLINT_NVTX_RANGE("flint_attn_layers_serial");
  const char* who = "flint_attn_layers_serial";
  if (!layers || !out) return fail(FLINT_ERR_INVALID_ARG, "%s: NULL pointer argument", who);
  if (n_layers < 1 || n_layers > FLINT_MAX_LAYERS)
    return fail(FLINT_ERR_INVALID_ARG, "%s: n_layers=%d outside [1, %d]", who, n_layers, FLINT_MAX_LAYERS);
  // One launch per layer, each after the first a programmatic dependent of
  // the one before: it waits for that launch to complete before it touches
  // memory, while its launch and set-up overlap the previous layer.
  for (int i = 0; i < n_layers; ++i) {
    flint_status s = run_stack(layers + i, 1, pos, eps, theta, out + static_cast<size_t>(i) * kHeads * kDim,
                               workspace, ws_bytes, num_ctas, dev_err, stream, i > 0 ? 1 : 0, who);
    if (s != FLINT_OK) return s;
  }
  return ok();
}

}  // extern "C"
