// flint_internal.h -- constants, kernel-parameter layout and launcher
// declarations shared by the CUDA sources of libflint.so.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <vector>

#include "flint.h"

// NVTX ranges around every entry point, for timelines in Nsight Systems or
// any NVTX consumer: compiled in with -DFLINT_NVTX (header-only NVTX 3, which
// costs nothing unless a tool is attached); release builds carry none.
#ifdef FLINT_NVTX
#include <nvtx3/nvToolsExt.h>
namespace flint {
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};
}  // namespace flint
#define FLINT_NVTX_RANGE(name) ::flint::NvtxRange flint_nvtx_range_(name)
#else
#define FLINT_NVTX_RANGE(name) ((void)0)
#endif

namespace flint {

constexpr int kHeads = FLINT_NUM_Q_HEADS;     // 32 query heads
constexpr int kKvHeads = FLINT_NUM_KV_HEADS;  // 4 KV heads
constexpr int kDim = FLINT_HEAD_DIM;          // 128
constexpr int kGroup = kHeads / kKvHeads;     // 8 query heads share a KV head
constexpr int kWindow = FLINT_WINDOW;         // 513
constexpr int kBlock = FLINT_BLOCK_SIZE;      // 64

// Decode pipeline geometry: a stage holds K and V of kTile tokens for all 4
// KV heads, as 16 TMA boxes of kTile rows x 64 dims (one per head, dim half
// and K/V), so a CTA reads whole 1 KiB token rows of the cache.  Taller boxes
// stream faster (measured: 32 rows ~4% above 16 rows).
#ifndef FLINT_TILE
#define FLINT_TILE 32
#endif
#ifndef FLINT_KV_EVICT_FIRST
#define FLINT_KV_EVICT_FIRST 1                // KV tiles loaded with an L2 evict-first hint
#endif
#ifndef FLINT_L2_PROMOTION
#define FLINT_L2_PROMOTION 3                  // CU_TENSOR_MAP_L2_PROMOTION_L2_256B
#endif
constexpr int kTile = FLINT_TILE;             // tokens per pipeline stage
constexpr int kBoxBytes = kTile * 64 * 2;     // one box: 2 KiB
constexpr int kBoxes = 2 * kKvHeads * 2;      // K/V x heads x dim halves = 16
constexpr int kStageBytes = kBoxes * kBoxBytes;  // 64 KiB at 32 tokens
#ifndef FLINT_STAGES
#define FLINT_STAGES 3
#endif
constexpr int kStages = FLINT_STAGES;
// Consumer warps come in groups of 4 (warp w of a group serves KV head w);
// every group takes part in every stage, group q on the q-th 16-token slice
// of the tile, so every warp waits on every stage's phases in order.  Two
// groups put two consumer warps on every scheduler.
constexpr int kSlice = 16;                    // tokens per consumer warp per stage
constexpr int kConsumerGroups = kTile / kSlice;
constexpr int kConsumerWarps = kKvHeads * kConsumerGroups;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
static_assert(kTile % kSlice == 0, "a tile splits into 16-token slices");

// Limits of one launch (bounded by the 32 KiB kernel-parameter space).
constexpr int kMaxProblems = 64;
constexpr int kMaxSegs = kMaxProblems;         // one segment per problem
constexpr int kMaxMaps = 2 * FLINT_MAX_LAYERS;
constexpr int kMaxItems = 768;
constexpr int kMaxCtas = 296;

// A problem split into more than kInlineMergeMax items is not merged by its
// last-arriving CTA (one CTA reading every partial would be the tail of the
// launch) but by the whole grid at the launch's end: after a grid barrier,
// or, for a problem over more than kWideMergeItems items, by the CTAs that
// finish streaming first as its items' ready flags come up.
constexpr int kInlineMergeMax = 16;

// A deferred problem with more partials than this is merged a CTA per unit
// (each of its 9 warps folding every 9th partial) instead of a warp per unit
// (the warp folding all partials).  So no warp folds more than
// kMergeWarpItems partials.
constexpr int kWideMergeItems = 96;
constexpr int kMergeWarpItems = 96;
static_assert(kWideMergeItems <= kMergeWarpItems && (kMaxItems + 8) / 9 <= kMergeWarpItems,
              "a merging warp folds at most kMergeWarpItems partials");

// One split partial of a problem: O for 32 heads (in the order the consumer
// warps hold it, chunk-interleaved across each warp's lanes), m [32] (log2
// units), l [32].
constexpr int kPartialFloats = kHeads * kDim + 2 * kHeads;
constexpr size_t kCounterBytes = 4096;
// int32 slots of the workspace's counter area: [0, kMaxSegs) per-problem
// arrival counters, then the grid-barrier word, the run-time queue head, the
// abort word and the merge-ticket word, and from kItemFlags one ready flag
// per item.
constexpr int kBarrierWord = kMaxSegs;
constexpr int kQueueHead = kMaxSegs + 1;
constexpr int kAbortWord = kMaxSegs + 2;
constexpr int kTicketWord = kMaxSegs + 3;
constexpr int kItemFlags = 128;
static_assert(kMaxItems % 32 == 0, "one raised-flag bit per item");
static_assert(kTicketWord < kItemFlags && kItemFlags + kMaxItems <= static_cast<int>(kCounterBytes / 4),
              "the counter area holds the counters and one flag per item");

// One attention problem: one request of one layer.
struct Problem {
  const void* q;            // q (bf16 or fp32, normed) or q_raw (bf16) when prep
  const uint16_t* k_raw;    // prep: bf16 [4][128]
  const uint16_t* v_raw;    // prep: bf16 [4][128]
  const uint16_t* w_q;      // prep: bf16 [128]
  const uint16_t* w_k;      // prep: bf16 [128]
  const float* sinks;       // fp32 [32]
  float* out;               // fp32 [32][128]
  uint16_t* k_rows;         // append target: this request's cache base (or the pool)
  uint16_t* v_rows;
  const int32_t* table;     // PAGED: this request's block-table row
  int32_t lo, hi;           // attended tokens [lo, hi) in storage coordinates
  int32_t tile_base;        // storage token of tile 0 (a multiple of 16 for PAGED)
  int32_t append_tok;       // storage-coordinate token of the new token, or -1
  int32_t pos;              // logical position of the new token (RoPE, paged append)
  int32_t num_blocks;       // PAGED pool size
  int32_t ext2, ext3;       // tensor extents along tokens and requests/blocks
  int32_t table_len;        // PAGED: entries in this request's block-table row
  int16_t map_k, map_v;     // tensor-map indices
  int16_t req;              // 4th tensor coordinate (request) for CONTIGUOUS/RING
  int8_t layout, q_fp32, rope;
  int8_t deferred;          // 1: merged at the launch's end (grid barrier or ready flags)
  int8_t fp8;               // 1: E4M3 cache, 64-token tiles, scales in kv_scales[map_k / 2]
  int8_t partial;           // 1: out receives the unnormalised partial (O [32][128], m [32],
                            //    l [32]; log2 units) and no sink is folded in (sinks may be NULL)
};
static_assert(sizeof(Problem) == 128, "Problem stays 128 bytes");

constexpr int kTileFp8 = 64;                  // tokens per stage for an E4M3 cache
constexpr int kBoxBytesFp8 = kTileFp8 * 128;  // one box: 128 dims x 64 tokens, 8 KiB

struct Item {
  int16_t seg;              // problem
  int16_t t0, t1;           // tile range within the problem's token range
  int16_t pad;
};

struct DecodeParams {
  CUtensorMap maps[kMaxMaps];
  Problem prob[kMaxProblems];
  Item items[kMaxItems];          // sorted by (problem, first tile)
  int16_t order[kMaxItems];       // static lists of the CTAs, then the run-time queue
  int16_t cta_item_begin[kMaxCtas + 1];  // CTA c's static items: order[begin[c] .. begin[c+1])
  int16_t seg_item_begin[kMaxSegs + 1];  // problem p's items: items[begin[p] .. begin[p+1])
  int32_t queue_begin;            // the queue is order[queue_begin .. queue_begin + n_queue)
  int32_t n_queue;
  int32_t* counters;        // workspace: per-segment arrival counters
  float* partials;          // workspace: one partial per item
  int32_t* dev_err;         // [0] status; debug builds also record a failed check in [2..7]
  float2 rope_cs[kDim / 2]; // prep: cos, sin of pos * theta^(-2i/128), from the host in double
  float kv_scales[kMaxMaps / 2][8];  // per cache (map pair): k_scale[4], v_scale[4] for E4M3
  float eps;
  int32_t n_problems;
  int32_t prep;             // 1: q/k norm (+RoPE) and append fused in (layer stack)
  int32_t n_items;          // items in the plan
  int32_t grid_merge;       // 1: the launch ends in a merge of the deferred problems
                            // (cooperative launch): some problem is deferred or the
                            // queue is not empty
  int16_t deferred[kMaxProblems];  // the deferred problems, those with many partials first
  int32_t n_deferred;
  int32_t n_wide;           // deferred[0, n_wide): merged a CTA per unit, the rest a warp per unit
  int32_t ws_items;         // partial slots in the workspace
  int32_t pdl;              // 1: programmatic dependent launch on the previous kernel of the
                            // stream: wait for it before touching global memory
  int32_t smem_bytes;       // dynamic shared memory of the launch
  int32_t merge_flags;      // 1: the merge at the launch's end runs on ready flags and
                            // tickets (decode_kernel<true>), 0: after a grid barrier
  uint32_t raised[kMaxItems / 32];  // bit i: item i is a deferred problem's (it raises a ready flag)
};

static_assert(sizeof(DecodeParams) <= 32000, "kernel parameters exceed 32 KiB");

struct PrepParams {
  const uint16_t* q_raw;
  const uint16_t* k_raw;
  const uint16_t* v_raw;
  const uint16_t* w_q;
  const uint16_t* w_k;
  float* q_out;
  uint16_t* k_out;
  // append target (k_rows == nullptr: no append)
  uint16_t* k_rows;
  uint16_t* v_rows;
  const int32_t* table;
  int64_t req_stride;
  int32_t layout, capacity, max_blocks, num_blocks;
  int32_t pos[kMaxProblems];
  int32_t* dev_err;
  double theta;
  float eps;
  int32_t apply_rope;
  int32_t do_norm;          // 0: k is already final (plain append)
  int32_t fp8;              // 1: E4M3 cache (k_rows / v_rows are byte rows)
  float k_scale[4], v_scale[4];
  // prefill (prefill_prep_kernel): token t of one prompt at position t, cache
  // request 0; a ring cache receives only the last `capacity` tokens
  int32_t prefill;
  int32_t n_tokens;
  uint16_t* q_out_bf16;     // q rounded to bf16 [T][32][128], or nullptr
  uint16_t* v_out_f16;      // v converted to fp16 [T][4][128] (saturating), or nullptr
};

// Prompt attention (prefill): q bf16 [T][32][128], k bf16 [T][4][128], v fp16
// [T][4][128], out fp32 [T][32][128]; query t attends keys
// max(0, t - window + 1) .. t (window > 0) or 0 .. t.
struct PrefillParams {
  // TMA maps, 128-byte swizzle, boxes of 64 dims:
  //   q_map  [128 dims][32 heads][T tokens][1], box 64 x 8 heads x 16 tokens
  //   k_map, v_map  [128 dims][4 heads][T tokens][1], box 64 x 1 x 128 tokens
  //   (k bf16, v fp16)
  CUtensorMap q_map, k_map, v_map;
  const float* sinks;
  float* out;
  int32_t* dev_err;
  int32_t T;
  int32_t window;
};

// A partial as the context-parallel calls exchange it: O [32][128] (natural
// dims), m [32], l [32], fp32.
constexpr int kCpPartialFloats = kHeads * kDim + 2 * kHeads;

// Launchers (return cudaGetLastError() after the launch).
cudaError_t launch_decode(const DecodeParams& p, int grid, cudaStream_t stream);  // cooperative if p.grid_merge
cudaError_t launch_prep(const PrepParams& p, int B, cudaStream_t stream);
// The prefill pass of one prompt (p.prefill = 1): a persistent grid of
// `grid` CTAs, each streaming a contiguous range of the p.n_tokens tokens.
int prefill_prep_grid(int T, int num_sms);
cudaError_t launch_prefill_prep(const PrepParams& p, int grid, cudaStream_t stream);
// One persistent CTA per SM (num_sms), each over a share of the (query block,
// KV head) units.
cudaError_t launch_prefill(const PrefillParams& p, int num_sms, cudaStream_t stream);
cudaError_t launch_merge_partials(const float* partials, int n_parts, int B, const float* sinks, float* out,
                                  cudaStream_t stream);

size_t decode_smem_bytes();

// Smallest workspace a launch of n_problems on num_ctas CTAs (0: one per SM)
// can run with: the counters and one partial per static item; 0 if invalid.
size_t workspace_min_bytes(int n_problems, int num_ctas);

// Sets the message that flint_last_error() returns on this thread; returns s.
flint_status record_error(flint_status s, const char* fmt, ...);

// The CUDA context current on the calling thread (a driver handle), or
// nullptr if there is none yet.  Per-context state (a kernel's shared-memory
// attribute, the address of a module variable) is keyed on it: after a device
// reset the runtime makes a new context, and state kept for the old one is void.
void* current_context();

// The contexts in which a kernel's launch attribute has been set.
struct ContextSet {
  std::mutex mu;
  std::vector<void*> ctxs;
};

// Sets the dynamic shared-memory limit of `kernel` to `bytes` once per
// context (thread-safe; `done` is the caller's record of configured contexts).
cudaError_t configure_once(ContextSet& done, const void* kernel, int bytes);

}  // namespace flint
