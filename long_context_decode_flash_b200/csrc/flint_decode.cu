// flint_decode.cu -- split-KV flash-decode for Flint's grouped-query attention
// with a per-head sink logit, on sm_100a.
//
// What is computed (page "Day-0 Support for Flint on vLLM", hnkhoi.com,
// "Model architecture": GQA 32 query / 4 KV heads, learned attention sinks,
// 513-token sliding window or full context): for query head h of KV group
// g = h / 8 and its token range R,
//     out_h = sum_{j in R} e^(s_j - M) V_j / (sum_{j in R} e^(s_j - M) + e^(sink_h - M)),
//     s_j = q_h . K_j / sqrt(128),  M = max(max_j s_j, sink_h).
//
// How (one persistent launch for every problem of the call):
//   * The host cuts each problem's token range into 32-token tiles and lays
//     most of them over one CTA per SM as static item lists (problem, tile
//     range; split-KV).  The tails of large problems are cut into chunks that
//     CTAs claim from a queue (atomic head in the workspace) once their own
//     lists are done, which evens out SMs that stream at different rates.
//   * The last warp is the producer: per 32-token tile it loads K and V of all
//     four KV heads with 16 TMA boxes (4-D tensor maps, 128-byte swizzle,
//     issued by lanes 0-15) into a 3-stage ring of 64 KiB stages guarded by
//     mbarriers, so the CTA reads whole 1 KiB token rows of the cache.  In the fused layer-stack
//     mode it first writes the new token's k (RMSNorm + RoPE) and v into the
//     cache, just before loading the tile that holds it.
//   * Consumer warps come in two groups of four; warp w of a group serves KV
//     head w and its 8 query heads, group q on the q-th 16-token half of
//     every tile, so every warp waits on every stage's phases in order (two
//     consumer warps per scheduler hide the MMA/softmax latency).  At an
//     item's end group 1 hands its state to group 0 through shared memory.
//     S^T = [q_hi; q_lo] K^T and O += [P_hi; P_lo] V run on bf16 mma.sync
//     m16n8k16, where the 16 rows of A are the 8 heads' hi and lo bf16 parts
//     (fp32 values split in two): the products carry ~16 significant bits
//     while K/V stay exact bf16.  Softmax runs in fp32 in log2 units with
//     quad shuffles; the running max moves only when it grows by more than 8
//     (warp-uniform branch), so rescales are rare.
//   * Item end: a problem covered by one item is finished on the spot (sink
//     folded in); otherwise the CTA stores a partial (m, l, O for 32 heads)
//     and the last CTA to arrive (atomic counter, no spinning) merges all
//     partials of the problem in item order and folds in the sinks.  A
//     problem split over many CTAs (more than kInlineMergeMax items) is
//     instead merged at the launch's end by the whole grid (cooperative
//     launch): after a grid barrier, or, for a problem over more than
//     kWideMergeItems items, by the CTAs that finish streaming first, each
//     batch of partials folded once its ready flags are up while the other
//     CTAs still stream.  Merge orders are fixed, so results are
//     deterministic.
// Every mbarrier wait is bounded in time; on timeout the kernel records
// FLINT_ERR_TIMEOUT, lets its loads land and returns.
#include <math.h>

#include "flint_device.cuh"

#ifndef FLINT_PREFETCH_MAPS
#define FLINT_PREFETCH_MAPS 0
#endif

namespace flint {

// Device-side timeline tracing, compiled in only with -DFLINT_TRACE: thread
// (0, lane 0 of a role) of every CTA stores %globaltimer at fixed points of
// its life into g_trace[block][slot]; flint_trace_read copies the table out.
// Release builds carry no trace code.
#ifdef FLINT_TRACE
constexpr int kTraceSlots = 16;
__device__ unsigned long long g_trace[kMaxCtas][kTraceSlots];
#define FLINT_TRACE_MARK(slot) (::flint::g_trace[blockIdx.x][(slot)] = ::flint::globaltimer_ns())
#define FLINT_TRACE_SET(slot, v) (::flint::g_trace[blockIdx.x][(slot)] = (v))
#else
#define FLINT_TRACE_MARK(slot) ((void)0)
#define FLINT_TRACE_SET(slot, v) ((void)0)
#endif

#ifdef FLINT_TEST_HOOKS
// {block, tile sequence number}: that CTA's producer leaves that tile's stage
// unarmed (no load, no expected bytes); {-1, -1} = off.
__device__ int g_stall_decode[2] = {-1, -1};
#endif

namespace {

// 2^x from the hardware unit (ex2.approx.ftz: ~2^-22 relative error, results
// below 2^-126 flushed to 0, which a softmax sum cannot tell apart).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

constexpr float kLog2e = 1.4426950408889634f;
// log2(e) / sqrt(128): scores come out of the tensor cores in log2 units.
constexpr float kQScale = static_cast<float>(1.4426950408889634 * 0.08838834764831845);
constexpr float kRescaleSlack = 8.0f;

// Per-thread state a consumer group hands to group 0 at an item's end:
// 32 O values, m, l.
constexpr int kXchFloats = 34;
constexpr int kXchSize = (kConsumerGroups - 1) * kKvHeads * 32 * kXchFloats;

// Small per-item inputs staged in shared memory one item ahead by the
// producer (bulk copies), so that neither the q set-up nor the new-token
// append waits on DRAM while the cache stream saturates it.
constexpr int kInQ = 0;          // q (bf16 [32][128]) or q_raw in the layer stack
constexpr int kInWq = 8192;      // w_q  bf16 [128]
constexpr int kInK = 8448;       // k_raw bf16 [4][128]
constexpr int kInV = 9472;       // v_raw bf16 [4][128]
constexpr int kInWk = 10496;     // w_k  bf16 [128]
constexpr int kInBytes = 10752;
constexpr int kAppendWarp = kConsumerWarps - 1;  // the consumer warp that appends

struct Smem {
  uint8_t* stages;
  uint64_t* full;
  uint64_t* empty;
  uint64_t* in_full;    // item inputs landed
  uint64_t* in_empty;   // item inputs consumed
  float2* cs;
  volatile int* flags;  // [0] abort, [1] last-arrival broadcast, [2] merge-ticket rank,
                        // [3] item whose new token is in the cache (+1),
                        // [4] item whose inputs are staged (producer -> consumers),
                        // [5] that item as consumer warp 0 saw it (-1: stop),
                        // [6] the launch's ready-flag value (merge tail)
  float* xch;           // group hand-over area
  uint8_t* in;          // item inputs
};

__device__ __forceinline__ Smem carve(uint8_t* raw) {
  Smem s;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  s.stages = base;
  s.full = reinterpret_cast<uint64_t*>(base + kStages * kStageBytes);
  s.empty = s.full + kStages;
  s.in_full = s.empty + kStages;
  s.in_empty = s.in_full + 1;
  s.cs = reinterpret_cast<float2*>(s.in_empty + 1);
  s.flags = reinterpret_cast<volatile int*>(s.cs + 64);
  s.xch = reinterpret_cast<float*>(s.cs + 64) + 8;
  s.in = reinterpret_cast<uint8_t*>(s.xch + kXchSize);  // 16-byte aligned
  return s;
}

// Byte offset of box (kv: 0 = K, 1 = V; head; dim half) inside a stage.
__device__ __forceinline__ uint32_t box_offset(int kv, int head, int half) {
  return static_cast<uint32_t>(((kv * kKvHeads + head) * 2 + half) * kBoxBytes);
}
// E4M3 stage: one box of 64 tokens x 128 dims per (K/V, head).
__device__ __forceinline__ uint32_t box_offset_fp8(int kv, int head) {
  return static_cast<uint32_t>((kv * kKvHeads + head) * kBoxBytesFp8);
}

__device__ __forceinline__ void consumer_bar() {
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
}

// Raise the CTA abort flag after a failed wait (timeout unless already aborted).
__device__ __forceinline__ void abort_cta(const DecodeParams& P, const Smem& S) {
  if (!S.flags[0]) report_error(P.dev_err, FLINT_ERR_TIMEOUT);
  S.flags[0] = 1;
}

// Ticket word, item flags and abort word of the merge at the launch's end
// (see merge_tail).
constexpr int kTicketShift = 12;
static_assert(2 * kMaxCtas < (1 << (kTicketShift - 1)), "ticket ranks stay apart from block 0's addend");

__device__ __forceinline__ unsigned int ld_relaxed_u32(const int32_t* p) {
  unsigned int v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_u32(int32_t* p, unsigned int v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Raises item `it`'s ready flag (thread 0, after the barrier that orders the
// other consumers' partial stores before it); `word` is the ticket word, read
// by the same thread at the item's end.
__device__ __forceinline__ void publish_item(const DecodeParams& P, int it, unsigned int word) {
  if (!FLINT_CHECK(P.dev_err, it >= 0 && it < P.n_items && it < kMaxItems, 9, it, P.n_items, 0)) return;
  st_release_u32(P.counters + kItemFlags + it, (word >> kTicketShift) + 1);
}

// Element offset, from the cache base the problem names, of the new token's
// row (all 4 heads); -1 if a paged block id is out of range.
__device__ __forceinline__ long long append_row(const Problem& pb) {
  if (pb.layout == FLINT_KV_PAGED) {
    const int blk = pb.table[pb.pos / kBlock];
    if (blk < 0 || blk >= pb.num_blocks) return -1;
    return (static_cast<long long>(blk) * kBlock + pb.pos % kBlock) * kKvHeads * kDim;
  }
  return static_cast<long long>(pb.append_tok) * kKvHeads * kDim;
}

// Fused layer stack, new token: norm (+RoPE) its k for every KV head from the
// staged inputs, round to bf16 and write it and v_raw into the cache; then
// order the writes before later TMA reads of those rows (async proxy).
__device__ void append_new_token(const DecodeParams& P, const Problem& pb, const uint8_t* in,
                                 int lane, const float2* cs) {
  const long long row = append_row(pb);
  if (row < 0) {
    if (lane == 0) report_error(P.dev_err, FLINT_ERR_INVALID_ARG);
    return;
  }
  const uint16_t* k_raw = reinterpret_cast<const uint16_t*>(in + kInK);
  const uint16_t* w_k = reinterpret_cast<const uint16_t*>(in + kInWk);
  const uint32_t* v_raw = reinterpret_cast<const uint32_t*>(in + kInV);
#pragma unroll
  for (int g = 0; g < kKvHeads; ++g) {
    float y[4];
    norm_rope_row_warp(k_raw + g * kDim, w_k, P.eps, true, pb.rope != 0, cs, lane, y);
    const uint32_t va = v_raw[g * 64 + lane], vb = v_raw[g * 64 + 32 + lane];
    if (!pb.fp8) {
      uint32_t* kd = reinterpret_cast<uint32_t*>(pb.k_rows + row + g * kDim);
      uint32_t* vd = reinterpret_cast<uint32_t*>(pb.v_rows + row + g * kDim);
      kd[lane] = pack_bf16x2(y[0], y[1]);
      kd[32 + lane] = pack_bf16x2(y[2], y[3]);
      vd[lane] = va;
      vd[32 + lane] = vb;
    } else {
      // E4M3: code = e4m3(x / scale), the division in float32 (IEEE, nearest)
      const float ks = P.kv_scales[pb.map_k >> 1][g], vs = P.kv_scales[pb.map_k >> 1][4 + g];
      uint16_t* kd = reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(pb.k_rows) + row + g * kDim);
      uint16_t* vd = reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(pb.v_rows) + row + g * kDim);
      kd[lane] = static_cast<uint16_t>(f32x2_to_e4m3x2(__fdiv_rn(y[0], ks), __fdiv_rn(y[1], ks)));
      kd[32 + lane] = static_cast<uint16_t>(f32x2_to_e4m3x2(__fdiv_rn(y[2], ks), __fdiv_rn(y[3], ks)));
      vd[lane] = static_cast<uint16_t>(f32x2_to_e4m3x2(__fdiv_rn(bf16_lo(va), vs), __fdiv_rn(bf16_hi(va), vs)));
      vd[32 + lane] = static_cast<uint16_t>(f32x2_to_e4m3x2(__fdiv_rn(bf16_lo(vb), vs), __fdiv_rn(bf16_hi(vb), vs)));
    }
  }
  fence_proxy_async_global();
}

// Producer: stage an item's small inputs (q or q_raw, norm weights, k_raw,
// v_raw) in shared memory with bulk copies completing on in_full.
__device__ __forceinline__ void issue_item_inputs(const DecodeParams& P, const Problem& pb,
                                                  const Smem& S) {
  const uint32_t fb = smem_u32(S.in_full);
  const uint32_t dst = smem_u32(S.in);
  if (P.prep) {
    mbar_expect_tx(fb, kInBytes);
    bulk_copy_g2s(dst + kInQ, pb.q, 8192, fb);
    bulk_copy_g2s(dst + kInWq, pb.w_q, 256, fb);
    bulk_copy_g2s(dst + kInK, pb.k_raw, 1024, fb);
    bulk_copy_g2s(dst + kInV, pb.v_raw, 1024, fb);
    bulk_copy_g2s(dst + kInWk, pb.w_k, 256, fb);
  } else if (!pb.q_fp32) {
    mbar_expect_tx(fb, 8192);
    bulk_copy_g2s(dst + kInQ, pb.q, 8192, fb);
  } else {
    mbar_arrive(fb);  // fp32 q is read from global memory
  }
}

// The next item of this CTA: its k-th static item, else a claim on the queue;
// -1 when there is no more work.
__device__ __forceinline__ int next_item(const DecodeParams& P, int k, int c0, int c1, bool claim) {
  if (c0 + k < c1) return P.order[c0 + k];
  if (!claim || P.n_queue <= 0) return -1;
  const int q = atomicAdd(P.counters + kQueueHead, 1);
  return q < P.n_queue ? P.order[P.queue_begin + q] : -1;
}

struct ProducerCount {
  int issued;  // tiles whose loads were issued
  int staged;  // in_full phases armed
};

__device__ ProducerCount run_producer(const DecodeParams& P, const Smem& S, int c0, int c1, bool claim,
                                      int lane) {
  int seq = 0;
  // lane i < 16 issues box i: K/V (i >> 3), head ((i >> 1) & 3), dim half (i & 1)
  const int my_kv = (lane >> 3) & 1, my_head = (lane >> 1) & 3, my_half = lane & 1;
#if FLINT_KV_EVICT_FIRST
  const uint64_t kv_policy = l2_policy_evict_first();
#endif
  for (int k = 0;; ++k) {
    int it = -1;
    {  // pick the next item once the consumers released the last inputs, and
       // stage its small inputs (or, with no item left, tell them to stop)
      bool ok = mbar_wait(smem_u32(S.in_empty), (static_cast<uint32_t>(k) & 1u) ^ 1u, S.flags);
      // once the CTA aborted, nothing more is staged or loaded
      ok = __all_sync(0xffffffffu, ok && !S.flags[0]);
      if (!ok) {
        if (lane == 0) abort_cta(P, S);
        return {seq, k};
      }
      if (lane == 0) {
        it = next_item(P, k, c0, c1, claim);
        if (!FLINT_CHECK(P.dev_err, it < P.n_items, 9, it, P.n_items, k)) it = -1;
        S.flags[4] = it;  // published by the arrive below (release)
        if (it >= 0)
          issue_item_inputs(P, P.prob[P.items[it].seg], S);
        else
          mbar_arrive(smem_u32(S.in_full));
      }
      it = __shfl_sync(0xffffffffu, it, 0);
      __syncwarp();
      if (it < 0) return {seq, k + 1};
    }
    const Item item = P.items[it];
    const Problem& pb = P.prob[item.seg];
    const bool fp8 = pb.fp8 != 0;
    const int tile_tok = fp8 ? kTileFp8 : kTile;
    // bf16: lane i < 16 loads box (K/V, head, dim half); E4M3: lane i < 8 loads box (K/V, head)
    const int b_kv = fp8 ? (lane >> 2) & 1 : my_kv, b_head = fp8 ? lane & 3 : my_head;
    const int n_boxes = fp8 ? 2 * kKvHeads : kBoxes;
    const uint32_t b_off = fp8 ? box_offset_fp8(b_kv, b_head) : box_offset(my_kv, my_head, my_half);
    const int b_x = fp8 ? 0 : 64 * my_half;
    const CUtensorMap* map = &P.maps[b_kv ? pb.map_v : pb.map_k];
    const bool paged = pb.layout == FLINT_KV_PAGED;
    const int app_tile = (P.prep && pb.append_tok >= 0) ? (pb.append_tok - pb.tile_base) / tile_tok : -1;
    for (int t = item.t0; t < item.t1; t += 32) {
      const int n = min(32, item.t1 - t);
      int blk = 0;
      if (paged && lane < n) {
        const int idx = (pb.tile_base + (t + lane) * tile_tok) / kBlock;
        if (FLINT_CHECK(P.dev_err, idx >= 0 && idx < pb.table_len, 3, idx, pb.table_len, it)) blk = __ldg(pb.table + idx);
        // A block id outside the pool: flag it for the caller; its tile's
        // loads are skipped below.
        if (blk < 0 || blk >= pb.num_blocks) report_error(P.dev_err, FLINT_ERR_INVALID_ARG);
      }
      for (int j = 0; j < n; ++j, ++seq) {
        const int b = __shfl_sync(0xffffffffu, blk, j);
        const int stage = seq % kStages;
        const uint32_t phase = static_cast<uint32_t>(seq / kStages) & 1u;
        bool ok = mbar_wait(smem_u32(&S.empty[stage]), phase ^ 1u, S.flags);
        // After an abort a consumer warp may have skipped a phase of this
        // stage, so the barrier's parity no longer says which tile it freed:
        // arm nothing more (the drain below waits for what was issued).
        ok = __all_sync(0xffffffffu, ok && !S.flags[0]);
        if (!ok) {
          if (lane == 0) abort_cta(P, S);
          return {seq, k + 1};
        }
        const int tile = t + j;
        if (tile == app_tile) {
          // the new token's rows are written by a consumer warp: wait for them
          bool done = true;
          if (lane == 0) {
            const unsigned long long t0 = globaltimer_ns();
            while (S.flags[3] != it + 1) {
              if (S.flags[0] || globaltimer_ns() - t0 > kWaitLimitNs) {
                done = false;
                break;
              }
            }
            __threadfence_block();
          }
          done = __shfl_sync(0xffffffffu, done, 0);
          if (!done) {
            if (lane == 0) abort_cta(P, S);
            return {seq, k + 1};
          }
        }
        const uint32_t fb = smem_u32(&S.full[stage]);
        const uint32_t base = smem_u32(S.stages + stage * kStageBytes);
        const int tok = pb.tile_base + tile * tile_tok;
        const int c2 = paged ? tok % kBlock : tok;
        const int c3 = paged ? b : pb.req;
        bool fine = true;
        if (lane == 0) {
          fine = FLINT_CHECK(P.dev_err, (base & 1023u) == 0 && base + kStageBytes <= smem_u32(S.full), 6,
                             static_cast<int>(base), stage, seq);
          // Every coordinate handed to TMA lies inside the tensor: a tile
          // outside it (only a bad paged block id can make one; reported
          // above) loads nothing.
          const bool in_range = c2 >= 0 && c2 < pb.ext2 && c3 >= 0 && c3 < pb.ext3;
          fine = fine && FLINT_CHECK(P.dev_err, in_range || paged, 5, c2, c3, it) && in_range;
#ifdef FLINT_TEST_HOOKS
          if (static_cast<int>(blockIdx.x) == g_stall_decode[0] && seq == g_stall_decode[1]) {
            fine = false;  // leave the stage unarmed: its waiters run out of time
          } else
#endif
          if (fine)
            mbar_expect_tx(fb, kStageBytes);
          else
            mbar_arrive(fb);  // complete the phase without data so nobody waits forever
        }
        fine = __shfl_sync(0xffffffffu, fine, 0);
        __syncwarp();
#ifdef FLINT_TRACE
        if (seq == 0 && lane == 0) FLINT_TRACE_MARK(2);
#endif
        if (fine && lane < n_boxes) {
#if FLINT_KV_EVICT_FIRST
          tma_load_4d_hint(base + b_off, map, fb, b_x, b_head, c2, c3, kv_policy);
#else
          tma_load_4d(base + b_off, map, fb, b_x, b_head, c2, c3);
#endif
        }
        __syncwarp();
      }
    }
  }
}

// Dims of the values a consumer thread with quad index c holds, 16 at a time:
// within each 16-dim chunk q, its values 0-1 are dims 16q + d0 + {0, 1} and
// values 2-3 are 16q + d2 + {0, 1}.  For a bf16 cache (d0, d2) = (2c, 2c + 8),
// the mma.sync fragment layout; for an E4M3 cache (4c, 4c + 2), the 4
// consecutive bytes ldmatrix gives a thread from a row of fp8 values.  The q
// fragment, the O accumulator and the outputs all follow the same map.
__device__ __forceinline__ int dim_d0(int c, bool fp8) { return fp8 ? 4 * c : 2 * c; }
__device__ __forceinline__ int dim_d2(int c, bool fp8) { return fp8 ? 4 * c + 2 : 2 * c + 8; }

// q fragments for query head h: thread (g = lane/4, c = lane%4) holds, for
// each 16-dim chunk kk, the dims above as the A operand rows g (hi part) and
// g + 8 (lo part), prescaled by log2(e)/sqrt(128); bf16 parts for a bf16
// cache, f16 parts for an E4M3 cache (the operands of one mma share a type).
__device__ __forceinline__ void load_q(const DecodeParams& P, const Problem& pb, const uint8_t* in,
                                       int h, int c, const float2* cs, uint32_t (&qa)[8][4]) {
  const bool fp8 = pb.fp8 != 0;
  const int d0 = dim_d0(c, fp8), d2 = dim_d2(c, fp8);
  float x[8][4];
  if (P.prep || !pb.q_fp32) {
    const uint16_t* q = reinterpret_cast<const uint16_t*>(in + kInQ) + h * kDim;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const uint32_t a = *reinterpret_cast<const uint32_t*>(q + 16 * kk + d0);
      const uint32_t b = *reinterpret_cast<const uint32_t*>(q + 16 * kk + d2);
      x[kk][0] = bf16_lo(a);
      x[kk][1] = bf16_hi(a);
      x[kk][2] = bf16_lo(b);
      x[kk][3] = bf16_hi(b);
    }
  } else {
    const float* q = static_cast<const float*>(pb.q) + h * kDim;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const float2 a = *reinterpret_cast<const float2*>(q + 16 * kk + d0);
      const float2 b = *reinterpret_cast<const float2*>(q + 16 * kk + d2);
      x[kk][0] = a.x;
      x[kk][1] = a.y;
      x[kk][2] = b.x;
      x[kk][3] = b.y;
    }
  }
  if (P.prep) {
    // per-head RMSNorm over the quad's 128 values, then RoPE pairs (i, i+64),
    // which sit in the same thread at kk and kk + 4
    float ss = 0.f;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
#pragma unroll
      for (int e = 0; e < 4; ++e) ss += x[kk][e] * x[kk][e];
    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
    ss += __shfl_xor_sync(0xffffffffu, ss, 2);
    const float r = 1.0f / sqrtf(ss * (1.0f / kDim) + P.eps);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const uint16_t* w_q = reinterpret_cast<const uint16_t*>(in + kInWq);
      const uint32_t a = *reinterpret_cast<const uint32_t*>(w_q + 16 * kk + d0);
      const uint32_t b = *reinterpret_cast<const uint32_t*>(w_q + 16 * kk + d2);
      x[kk][0] = x[kk][0] * r * bf16_lo(a);
      x[kk][1] = x[kk][1] * r * bf16_hi(a);
      x[kk][2] = x[kk][2] * r * bf16_lo(b);
      x[kk][3] = x[kk][3] * r * bf16_hi(b);
    }
    if (pb.rope) {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 t = cs[16 * kk + ((e >> 1) ? d2 : d0) + (e & 1)];
          const float a = x[kk][e], b = x[kk + 4][e];
          x[kk][e] = a * t.x - b * t.y;
          x[kk + 4][e] = b * t.x + a * t.y;
        }
    }
  }
  if (fp8) {
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      split_f16x2(x[kk][0] * kQScale, x[kk][1] * kQScale, qa[kk][0], qa[kk][1]);
      split_f16x2(x[kk][2] * kQScale, x[kk][3] * kQScale, qa[kk][2], qa[kk][3]);
    }
  } else {
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      split_bf16x2(x[kk][0] * kQScale, x[kk][1] * kQScale, qa[kk][0], qa[kk][1]);
      split_bf16x2(x[kk][2] * kQScale, x[kk][3] * kQScale, qa[kk][2], qa[kk][3]);
    }
  }
}

// One 16-token slice of a tile for KV head w and its 8 query heads: online-
// softmax update of (m_run, l_run, o).  sK / sV point at row r0 of the head's
// 64-dim K / V boxes (kTile rows of 128 bytes each, 128-byte swizzle, r0 a
// multiple of 8); tok0 is the storage token of that row.
__device__ __forceinline__ void consume_slice(uint32_t sK, uint32_t sV, int tok0, int lo, int hi,
                                              int lane, const uint32_t (&qa)[8][4], float& m_run,
                                              float& l_run, float (&o)[16][4]) {
  const int c = lane & 3;
  const int l7 = lane & 7;
  const bool whole = (tok0 >= lo) && (tok0 + kSlice <= hi);

  // S^T = [q_hi; q_lo] * K^T: 2 n-tiles of 8 tokens, 8 k-steps of 16 dims.
  // (two accumulators per n-tile keep the dependent MMA chains short)
  float sc[4];
#pragma unroll
  for (int jj = 0; jj < 2; ++jj) {
    float a0[4] = {0.f, 0.f, 0.f, 0.f}, a1[4] = {0.f, 0.f, 0.f, 0.f};
    const uint32_t row = sK + (8 * jj + l7) * 128;
#pragma unroll
    for (int kk = 0; kk < 8; kk += 2) {
      const int u = 2 * kk + (lane >> 3);  // 16-byte unit along the 128 dims
      uint32_t b0, b1, b2, b3;
      ldsm_x4(row + (u >> 3) * kBoxBytes + (((u & 7) ^ l7) << 4), b0, b1, b2, b3);
      mma_bf16_16816(a0, qa[kk], b0, b1);
      mma_bf16_16816(a1, qa[kk + 1], b2, b3);
    }
    // rows g (q hi part) and g + 8 (q lo part): token tok0 + 8jj + 2c (+1)
    sc[2 * jj] = (a0[0] + a1[0]) + (a0[2] + a1[2]);
    sc[2 * jj + 1] = (a0[1] + a1[1]) + (a0[3] + a1[3]);
  }
  if (!whole) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int tok = tok0 + 8 * (i >> 1) + 2 * c + (i & 1);
      if (tok < lo || tok >= hi) sc[i] = -INFINITY;
    }
  }

  float mx = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
  // The running max moves only when a head's max grows by more than the
  // slack (always on its first valid tile); the branch is warp-uniform.
  const bool grow = mx > m_run + kRescaleSlack;
  if (__any_sync(0xffffffffu, grow)) {
    const float alpha = grow ? ex2_approx(m_run - mx) : 1.0f;
    l_run *= alpha;
#pragma unroll
    for (int n = 0; n < 16; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[n][e] *= alpha;
    if (grow) m_run = mx;
  }
  const float mu = (m_run == -INFINITY) ? 0.f : m_run;

  // P = 2^(s - m) split into the bf16 hi/lo rows of the A operand.
  const float p0 = ex2_approx(sc[0] - mu), p1 = ex2_approx(sc[1] - mu);
  const float p2 = ex2_approx(sc[2] - mu), p3 = ex2_approx(sc[3] - mu);
  l_run += (p0 + p1) + (p2 + p3);
  uint32_t pa[4];
  split_bf16x2(p0, p1, pa[0], pa[1]);
  split_bf16x2(p2, p3, pa[2], pa[3]);

  // O += [P_hi; P_lo] * V: one k-step of 16 tokens, 16 n-tiles of 8 dims.
  uint32_t m01 = 0xffffffffu, m23 = 0xffffffffu;
  if (!whole) {
    const int t = tok0 + 2 * c;
    m01 = ((t >= lo && t < hi) ? 0x0000ffffu : 0u) | ((t + 1 >= lo && t + 1 < hi) ? 0xffff0000u : 0u);
    m23 = ((t + 8 >= lo && t + 8 < hi) ? 0x0000ffffu : 0u) |
          ((t + 9 >= lo && t + 9 < hi) ? 0xffff0000u : 0u);
  }
  const uint32_t row = sV + (((lane >> 3) & 1) * 8 + l7) * 128;
#pragma unroll
  for (int np = 0; np < 8; ++np) {
    const int nt = 2 * np + (lane >> 4);
    uint32_t v0, v1, v2, v3;
    ldsm_x4_t(row + (nt >> 3) * kBoxBytes + (((nt & 7) ^ l7) << 4), v0, v1, v2, v3);
    if (!whole) {  // rows outside the range may hold anything (even NaN)
      v0 &= m01;
      v2 &= m01;
      v1 &= m23;
      v3 &= m23;
    }
    mma_bf16_16816(o[2 * np], pa, v0, v1);
    mma_bf16_16816(o[2 * np + 1], pa, v2, v3);
  }
}

// The E4M3 counterpart of consume_slice, for a 32-token block (one softmax
// step for the block).  sK / sV point at row r0 of the head's K / V boxes
// (kTileFp8 rows of 128 one-byte dims, 128-byte swizzle, r0 a multiple of 8).
//   * QK: ldmatrix gives thread (g, c) 4 consecutive bytes of a row (dims
//     16u + 4c .. 16u + 4c + 3), widened to f16: the B fragment of K^T for
//     the logical k order q was loaded in (d0 = 4c, d2 = 4c + 2).  Scores
//     are then multiplied by the head's k scale.
//   * PV: ldmatrix.trans on byte pairs gives a thread tokens 2c, 2c + 1 of
//     dims 2p, 2p + 1 (p = g) of a 16-dim chunk; one byte permute splits them
//     into the B fragments of the chunk's even-dim and odd-dim n-tiles.  O
//     n-tile 2u holds dims 16u + 4c + {0, 2} and n-tile 2u + 1 dims
//     16u + 4c + {1, 3} of thread (g, c) (see fp8_o_to_values).
// The caller multiplies O by the head's v scale at the item's end.  kWhole:
// every token of the block lies in [lo, hi), so no row needs a mask (the
// caller picks the instance; the masks are ALU work on every value).
template <bool kWhole>
__device__ __forceinline__ void consume_block32_fp8(uint32_t sK, uint32_t sV, int tok0, int lo, int hi,
                                                    int lane, const uint32_t (&qa)[8][4], float k_scale,
                                                    float& m_run, float& l_run, float (&o)[16][4]) {
  const int c = lane & 3;
  const int l7 = lane & 7;
  constexpr bool whole = kWhole;

  float sc[8];
#pragma unroll
  for (int jj = 0; jj < 4; ++jj) {
    float a0[4] = {0.f, 0.f, 0.f, 0.f}, a1[4] = {0.f, 0.f, 0.f, 0.f};
    const uint32_t row = sK + (8 * jj + l7) * 128;
#pragma unroll
    for (int kk = 0; kk < 8; kk += 4) {
      const int u = kk + (lane >> 3);  // lanes 8i..8i+7 address 16-dim chunk kk + i
      uint32_t r[4];
      ldsm_x4(row + ((u ^ l7) << 4), r[0], r[1], r[2], r[3]);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint32_t b0, b1;
        e4m3x4_to_f16x2x2(r[i], b0, b1);
        if (i & 1)
          mma_f16_16816(a1, qa[kk + i], b0, b1);
        else
          mma_f16_16816(a0, qa[kk + i], b0, b1);
      }
    }
    // rows g (q hi) and g + 8 (q lo) of both accumulators, two tokens at a time
    const float2 t = add2(add2(make_float2(a0[0], a0[1]), make_float2(a1[0], a1[1])),
                          add2(make_float2(a0[2], a0[3]), make_float2(a1[2], a1[3])));
    const float2 st = mul2(t, make_float2(k_scale, k_scale));
    sc[2 * jj] = st.x;
    sc[2 * jj + 1] = st.y;
  }
  if (!whole) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int tok = tok0 + 8 * (i >> 1) + 2 * c + (i & 1);
      if (tok < lo || tok >= hi) sc[i] = -INFINITY;
    }
  }

  float mx = sc[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) mx = fmaxf(mx, sc[i]);
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
  const bool grow = mx > m_run + kRescaleSlack;
  if (__any_sync(0xffffffffu, grow)) {
    const float alpha = grow ? ex2_approx(m_run - mx) : 1.0f;
    l_run *= alpha;
#pragma unroll
    for (int n = 0; n < 16; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[n][e] *= alpha;
    if (grow) m_run = mx;
  }
  const float mu = (m_run == -INFINITY) ? 0.f : m_run;

  float p[8];
  const float2 nmu = make_float2(-mu, -mu);
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    const float2 x = add2(make_float2(sc[i], sc[i + 1]), nmu);
    p[i] = ex2_approx(x.x);
    p[i + 1] = ex2_approx(x.y);
  }
  {
    const float2 s01 = add2(add2(make_float2(p[0], p[1]), make_float2(p[2], p[3])),
                            add2(make_float2(p[4], p[5]), make_float2(p[6], p[7])));
    l_run += s01.x + s01.y;
  }
  uint32_t pa[2][4];  // k-steps of 16 tokens
#pragma unroll
  for (int s2 = 0; s2 < 2; ++s2) {
    split_f16x2(p[4 * s2], p[4 * s2 + 1], pa[s2][0], pa[s2][1]);
    split_f16x2(p[4 * s2 + 2], p[4 * s2 + 3], pa[s2][2], pa[s2][3]);
  }

  // masks of a thread's token pairs (2c, 2c + 1) + 8 i, i = 0..3
  uint32_t msk[4] = {0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu};
  if (!whole) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int t = tok0 + 8 * i + 2 * c;
      msk[i] = ((t >= lo && t < hi) ? 0x0000ffffu : 0u) | ((t + 1 >= lo && t + 1 < hi) ? 0xffff0000u : 0u);
    }
  }
  // lanes 8i..8i+7 address tokens 8i + l7 of the chunk (all four 8-token groups)
  const uint32_t row = sV + (8 * (lane >> 3) + l7) * 128;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    uint32_t x[4];
    ldsm_x4_t(row + ((u ^ l7) << 4), x[0], x[1], x[2], x[3]);
    uint32_t ev[4], od[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      // x[i]: bytes (t 2c: d 2g, d 2g+1), (t 2c+1: d 2g, d 2g+1) of token group i
      const uint32_t y = __byte_perm(x[i], 0u, 0x3120);  // (t2c d2g, t2c+1 d2g, t2c d2g+1, t2c+1 d2g+1)
      e4m3x4_to_f16x2x2(y, ev[i], od[i]);               // dims 2g, 2g+1 of tokens 2c, 2c+1
      if (!whole) {
        ev[i] &= msk[i];
        od[i] &= msk[i];
      }
    }
#pragma unroll
    for (int s2 = 0; s2 < 2; ++s2) {
      mma_f16_16816(o[2 * u], pa[s2], ev[2 * s2], ev[2 * s2 + 1]);
      mma_f16_16816(o[2 * u + 1], pa[s2], od[2 * s2], od[2 * s2 + 1]);
    }
  }
}

// The 32 O values of thread (g, c) in the order of the dim map (values 4q..4q+3
// = dims 16q + 4c + 0..3), from consume_block32_fp8's accumulators, rows g
// (P hi) and g + 8 (P lo) summed.
__device__ __forceinline__ void fp8_o_to_values(const float (&o)[16][4], float scale, float (&v)[32]) {
#pragma unroll
  for (int q = 0; q < 8; ++q)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      v[4 * q + 2 * e] = (o[2 * q][e] + o[2 * q][e + 2]) * scale;          // even n-tile: dim 4c + 2e
      v[4 * q + 2 * e + 1] = (o[2 * q + 1][e] + o[2 * q + 1][e + 2]) * scale;  // odd: 4c + 2e + 1
    }
}

// Float4 slot of values 4q..4q+3 of consumer thread (head, c)'s 32 O values
// inside a partial.  The 32 threads of a KV head's warp (lane = 4(head % 8) + c)
// hold chunk q in 512 consecutive bytes, so a warp's load or store of one
// chunk touches 4 cache lines, not 32.
__device__ __forceinline__ int partial_f4(int head, int c, int q) {
  return ((head >> 3) * 8 + q) * 32 + (head & 7) * 4 + c;
}

// The factor that turns an unnormalised O (with running max M and sum L, log2
// units) into the output with the head's sink logit folded into the softmax:
// 2^(M - Mf) / (L 2^(M - Mf) + 2^(s - Mf)), s = sink log2(e), Mf = max(M, s).
// With no key (M = -inf) the output is 0, whatever the sink (also for a sink
// of -inf, where the formula would read 0/0).
__device__ __forceinline__ float sink_scale(float M, float L, float sink) {
  if (M == -INFINITY) return 0.f;
  const float s2 = sink * kLog2e;
  const float Mf = fmaxf(M, s2);
  const float a = exp2f(M - Mf);
  return a / (L * a + exp2f(s2 - Mf));
}

// out[head][8n + 2c + e] = O * 2^(M - Mf) / (L 2^(M - Mf) + 2^(sink - Mf)), the
// sink logit of this head folded into the softmax; thread (g, c) owns dims
// 8n + 2c + {0,1} of head `head`.
__device__ __forceinline__ void finish_head(const Problem& pb, int head, int c, float M, float L,
                                            const float (&v)[32], float sink) {
  if (pb.partial) {
    // unnormalised partial for a later merge across ranks: O, m, l
    float* dst = pb.out + head * kDim;
    const int d0 = dim_d0(c, pb.fp8 != 0), d2 = dim_d2(c, pb.fp8 != 0);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      *reinterpret_cast<float2*>(dst + 16 * q + d0) = make_float2(v[4 * q], v[4 * q + 1]);
      *reinterpret_cast<float2*>(dst + 16 * q + d2) = make_float2(v[4 * q + 2], v[4 * q + 3]);
    }
    if (c == 0) {
      pb.out[kHeads * kDim + head] = M;
      pb.out[kHeads * kDim + kHeads + head] = L;
    }
    return;
  }
  const float scale = sink_scale(M, L, sink);
  float* dst = pb.out + head * kDim;
  const int d0 = dim_d0(c, pb.fp8 != 0), d2 = dim_d2(c, pb.fp8 != 0);
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    *reinterpret_cast<float2*>(dst + 16 * q + d0) = make_float2(v[4 * q] * scale, v[4 * q + 1] * scale);
    *reinterpret_cast<float2*>(dst + 16 * q + d2) = make_float2(v[4 * q + 2] * scale, v[4 * q + 3] * scale);
  }
}

// Folds partials i = s0 + r, s0 + r + stride, ... (< s1) of (head, quarter c)
// into a running (m, l, v), in increasing i.
__device__ __forceinline__ void fold_partials(const DecodeParams& P, int s0, int s1, int r, int stride,
                                              int head, int c, float& m, float& l, float (&v)[32]) {
  // two partials per round, both loaded before either is folded
  for (int i = s0 + r; i < s1; i += 2 * stride) {
    float mi[2], li[2];
    float4 ov[2][8];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int ij = i + j * stride;
      const float* pi = P.partials + static_cast<size_t>(ij < s1 ? ij : i) * kPartialFloats;
      mi[j] = ij < s1 ? __ldcg(pi + kHeads * kDim + head) : -INFINITY;
      li[j] = __ldcg(pi + kHeads * kDim + kHeads + head);
      const float4* po = reinterpret_cast<const float4*>(pi);
#pragma unroll
      for (int q = 0; q < 8; ++q) ov[j][q] = __ldcg(po + partial_f4(head, c, q));
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const float mn = fmaxf(m, mi[j]);
      const float sa = (m == -INFINITY) ? 0.f : exp2f(m - mn);
      const float sb = (mi[j] == -INFINITY) ? 0.f : exp2f(mi[j] - mn);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        v[4 * q] = v[4 * q] * sa + ov[j][q].x * sb;
        v[4 * q + 1] = v[4 * q + 1] * sa + ov[j][q].y * sb;
        v[4 * q + 2] = v[4 * q + 2] * sa + ov[j][q].z * sb;
        v[4 * q + 3] = v[4 * q + 3] * sa + ov[j][q].w * sb;
      }
      l = l * sa + li[j] * sb;
      m = mn;
    }
  }
}

template <bool kFlags>
__device__ void run_consumer(const DecodeParams& P, const Smem& S, int warp, int lane) {
  const int g = lane >> 2, c = lane & 3;
  const int kvh = warp % kKvHeads;      // the KV head this warp serves
  const int group = warp / kKvHeads;    // its consumer group
  const int head = kvh * kGroup + g;    // the query head this thread's quad serves
  int seq = 0;
  for (int k = 0;; ++k) {
    uint32_t qa[8][4];
    // Every consumer warp waits for the staged inputs itself; all of them
    // then take the item as warp 0 saw it, so they agree on when to stop and
    // meet the same barriers.  Warp 0 rewrites flags[5] only once the next
    // inputs are staged, which needs every warp's in_empty arrival below,
    // made after its read (and the item-end barriers come in between too).
    bool ok = mbar_wait(smem_u32(S.in_full), static_cast<uint32_t>(k) & 1u, S.flags);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok && lane == 0) abort_cta(P, S);
    if (warp == 0 && lane == 0) S.flags[5] = ok ? S.flags[4] : -1;
    consumer_bar();
    const int it = S.flags[5];
    if (it < 0) break;
    const Item item = P.items[it];
    const Problem& pb = P.prob[item.seg];
    // this head's sink logit, needed only at the item's end: load it now
    const float sink = pb.sinks ? pb.sinks[head] : 0.f;
    // E4M3 cache: the KV head's scales (unused for bf16)
    const float k_scale = P.kv_scales[pb.map_k >> 1][kvh];
    const float v_scale = P.kv_scales[pb.map_k >> 1][4 + kvh];
    {
      load_q(P, pb, S.in, head, c, S.cs, qa);
      if (P.prep && warp == kAppendWarp && pb.append_tok >= 0) {
        const int app_tile = (pb.append_tok - pb.tile_base) / (pb.fp8 ? kTileFp8 : kTile);
        if (app_tile >= item.t0 && app_tile < item.t1) {
          append_new_token(P, pb, S.in, lane, S.cs);
          __syncwarp();
          if (lane == 0) {
            __threadfence_block();
            S.flags[3] = it + 1;
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(S.in_empty));
    }

    float m_run = -INFINITY, l_run = 0.f;
    float o[16][4];
#pragma unroll
    for (int n = 0; n < 16; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[n][e] = 0.f;

    const int ntiles = item.t1 - item.t0;
    for (int k = 0; k < ntiles; ++k, ++seq) {
      // Once the CTA aborted, a warp neither waits, reads nor releases a
      // stage: a warp that gave up on a phase would otherwise pass the parity
      // wait of the same stage's next tile on an older phase.  It keeps
      // walking so that every warp meets the same barriers.
      if (__any_sync(0xffffffffu, S.flags[0] != 0)) continue;
      const int stage = seq % kStages;
      const uint32_t phase = static_cast<uint32_t>(seq / kStages) & 1u;
      // every lane observes the phase completion (acquire) before reading the stage
      bool ok = mbar_wait(smem_u32(&S.full[stage]), phase, S.flags);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        if (lane == 0) abort_cta(P, S);
        continue;
      }
#ifdef FLINT_TRACE
      if (seq == 0 && warp == 0 && lane == 0) FLINT_TRACE_MARK(3);
#endif
      const uint32_t base = smem_u32(S.stages + stage * kStageBytes);
      if (!pb.fp8) {
        const int r0 = group * kSlice;
        const int tok0 = pb.tile_base + (item.t0 + k) * kTile + r0;
        consume_slice(base + box_offset(0, kvh, 0) + r0 * 128, base + box_offset(1, kvh, 0) + r0 * 128,
                      tok0, pb.lo, pb.hi, lane, qa, m_run, l_run, o);
      } else {
        // 64-token E4M3 tile: group q takes tokens 32q .. 32q + 31 as one block
        const int r0 = group * (kTileFp8 / kConsumerGroups);
        const int tok0 = pb.tile_base + (item.t0 + k) * kTileFp8 + r0;
        if (tok0 >= pb.lo && tok0 + 32 <= pb.hi)
          consume_block32_fp8<true>(base + box_offset_fp8(0, kvh) + r0 * 128,
                                    base + box_offset_fp8(1, kvh) + r0 * 128, tok0, pb.lo, pb.hi, lane, qa,
                                    k_scale, m_run, l_run, o);
        else
          consume_block32_fp8<false>(base + box_offset_fp8(0, kvh) + r0 * 128,
                                     base + box_offset_fp8(1, kvh) + r0 * 128, tok0, pb.lo, pb.hi, lane, qa,
                                     k_scale, m_run, l_run, o);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&S.empty[stage]));
    }

    // ---- item end: this warp holds (m, l, O) of its 8 heads over the item
    if (warp == 0 && lane == 0) FLINT_TRACE_MARK(4);
    // ready-flag mode: the epoch for a deferred item's flag, read now so that
    // the load is in flight while the partial is stored
    [[maybe_unused]] unsigned int ticket_word = 0u;
    if constexpr (kFlags) {
      if (pb.deferred && threadIdx.x == 0) ticket_word = ld_relaxed_u32(P.counters + kTicketWord);
    }
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
    float v[32];
    if (pb.fp8) {
      fp8_o_to_values(o, v_scale, v);  // E4M3: V was read as codes
    } else {
#pragma unroll
      for (int n = 0; n < 16; ++n) {
        v[2 * n] = o[n][0] + o[n][2];
        v[2 * n + 1] = o[n][1] + o[n][3];
      }
    }
    if (kConsumerGroups > 1) {
      // the other groups hand their states to group 0, which merges them
      float* mine = S.xch + ((group - 1) * kKvHeads * 32 + kvh * 32 + lane) * kXchFloats;
      if (group > 0) {
#pragma unroll
        for (int e = 0; e < 32; ++e) mine[e] = v[e];
        mine[32] = m_run;
        mine[33] = l_run;
      }
      __syncwarp();
      consumer_bar();
      if (group == 0) {
#pragma unroll 1
        for (int q = 1; q < kConsumerGroups; ++q) {
          const float* other = S.xch + ((q - 1) * kKvHeads * 32 + kvh * 32 + lane) * kXchFloats;
          const float mo = other[32], lo_ = other[33];
          const float M = fmaxf(m_run, mo);
          const float sa = (m_run == -INFINITY) ? 0.f : exp2f(m_run - M);
          const float sb = (mo == -INFINITY) ? 0.f : exp2f(mo - M);
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = v[e] * sa + other[e] * sb;
          l_run = l_run * sa + lo_ * sb;
          m_run = M;
        }
      }
    }
    const int s0 = P.seg_item_begin[item.seg], s1 = P.seg_item_begin[item.seg + 1];
    if (s1 - s0 == 1) {
      if (group == 0) finish_head(pb, head, c, m_run, l_run, v, sink);
      __syncwarp();
      consumer_bar();  // the hand-over area is reused by the next item
      continue;
    }
    float* part = P.partials + static_cast<size_t>(it) * kPartialFloats;
    if (group == 0 &&
        FLINT_CHECK(P.dev_err, it < P.ws_items && s0 >= 0 && s1 <= P.n_items, 7, it, s0, s1)) {
      float4* pd = reinterpret_cast<float4*>(part);
#pragma unroll
      for (int q = 0; q < 8; ++q)
        pd[partial_f4(head, c, q)] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
      if (c == 0) {
        part[kHeads * kDim + head] = m_run;
        part[kHeads * kDim + kHeads + head] = l_run;
      }
    }
    __syncwarp();
    consumer_bar();
    if (threadIdx.x == 0) FLINT_TRACE_MARK(5);
    // One thread releases the partial (the barrier above orders every
    // consumer's stores before it).  A deferred problem's item raises its
    // ready flag for the CTAs that merge at the launch's end (ready-flag
    // mode) or waits for the grid barrier; otherwise the thread counts the
    // arrival, and the last CTA to arrive merges.
    if (pb.deferred) {
      if constexpr (kFlags) {
        if (threadIdx.x == 0) {
          publish_item(P, it, ticket_word);
          FLINT_TRACE_MARK(12);
        }
      }
      continue;
    }
    if (threadIdx.x == 0) {
      int prev = 0;
      __threadfence();
      if (FLINT_CHECK(P.dev_err, item.seg < kMaxSegs, 8, item.seg, 0, 0))
        prev = atomicAdd(P.counters + item.seg, 1);
      __threadfence();
      S.flags[1] = (prev == s1 - s0 - 1) ? 1 : 0;
    }
    consumer_bar();
    if (S.flags[1]) {
      // last arrival: both groups fold half of the problem's partials each
      // (items s0 + group, s0 + group + 2, ...; two loads in flight per
      // thread), then group 1 hands its state to group 0, which finishes
      float mm = -INFINITY, ll = 0.f;
#pragma unroll
      for (int e = 0; e < 32; ++e) v[e] = 0.f;
      fold_partials(P, s0, s1, group, kConsumerGroups, head, c, mm, ll, v);
      float* mine = S.xch + (kvh * 32 + lane) * kXchFloats;
      if (group == 1) {
#pragma unroll
        for (int e = 0; e < 32; ++e) mine[e] = v[e];
        mine[32] = mm;
        mine[33] = ll;
      }
      __syncwarp();
      consumer_bar();
      if (group == 0) {
        const float mo = mine[32], lo_ = mine[33];
        const float M = fmaxf(mm, mo);
        const float sa = (mm == -INFINITY) ? 0.f : exp2f(mm - M);
        const float sb = (mo == -INFINITY) ? 0.f : exp2f(mo - M);
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = v[e] * sa + mine[e] * sb;
        finish_head(pb, head, c, M, ll * sa + lo_ * sb, v, sink);
        if (threadIdx.x == 0) P.counters[item.seg] = 0;  // ready for the next call
        if (threadIdx.x == 0) FLINT_TRACE_MARK(12);
      }
    }
    __syncwarp();
    consumer_bar();  // flags[1] and the hand-over area are reused by the next item
  }
}

// ---- merge of the deferred problems at the launch's end --------------------
// Two modes, chosen per launch by the planner (P.merge_flags):
//   * Grid barrier (0): every CTA arrives once its streaming is over; then
//     CTA b merges tasks b, b + G, ...  Cheapest where the CTAs end together
//     (short streams, or the run-time queue evening out the end).
//   * Ready flags (1, when a problem is split over more than kWideMergeItems
//     items): the CTAs that finish streaming first merge while the others
//     still stream, each batch of partials once its items' flags are up.  It
//     pays where the CTAs' end times spread over microseconds (a lone long
//     context: ~21 tiles per CTA, SMs differing by up to ~28 % in rate).
//     Its protocol:
//   * Ticket (counters[kTicketWord]): after its streaming every CTA takes
//     exactly one.  Block 0 adds 2^12 - (G - 1), the others add 1, so the
//     low 12 bits return to zero once all G CTAs took theirs, and the carry
//     out of them counts launches in bits 12..31: the launch's epoch E, the
//     same in every CTA's ticket.  A CTA's rank is the number of tickets
//     taken before its own; rank r merges tasks r, r + G, ...
//   * Item flags (counters[kItemFlags + item]): after the consumers' barrier
//     at the item's end, thread 0 stores E + 1 with release order.  It reads
//     E from the ticket word (the load issued as the item ends, so that it is
//     in flight while the partial is stored): no carry can happen before this
//     CTA takes its own ticket.
//   * Abort word (counters[kAbortWord]): a CTA that aborted stores E + 1, so
//     that the merging CTAs stop waiting for its items.
//   * The CTA of rank G - 1 knows that every CTA has made its last claim and
//     raised its last flag: it resets the queue head and zeroes every flag
//     this launch did not raise.  So at a launch's start each flag holds zero
//     or the previous such launch's value (E), never this launch's E + 1,
//     whatever the plans of earlier launches were.
#ifndef FLINT_MERGE_BATCH
#define FLINT_MERGE_BATCH 8
#endif
constexpr int kMergeBatch = FLINT_MERGE_BATCH;
// Takes this CTA's ticket (thread 0): returns its rank, sets *ready = E + 1.
__device__ __forceinline__ int take_ticket(const DecodeParams& P, unsigned int* ready) {
  const unsigned int G = gridDim.x;
  const unsigned int add = blockIdx.x == 0 ? (1u << kTicketShift) - (G - 1) : 1u;
  unsigned int old;
  // acquire: the queue reset by the last ticket's CTA follows every other
  // CTA's claims; release: this CTA's claims precede its ticket
  asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], %2;"
               : "=r"(old)
               : "l"(P.counters + kTicketWord), "r"(add)
               : "memory");
  *ready = (old >> kTicketShift) + 1;
  const unsigned int lo = old & ((1u << kTicketShift) - 1);
  if (blockIdx.x == 0 || lo < (1u << (kTicketShift - 1))) return static_cast<int>(lo);
  return static_cast<int>(lo + G) - (1 << kTicketShift);  // block 0 came before
}

// The merge works in units of (problem, KV head g, chunk q).  Lane (h, c) of
// a warp owns values 4q..4q+3 of head 8g + h, quarter c: dims 16q + d0 +
// {0, 1} and 16q + d2 + {0, 1} of the head (see dim_d0; the layout the
// consumer warps wrote), so one warp load reads 512 consecutive bytes of a
// partial.  A lane folds its partials kMergeBatch loads at a time, a batch
// once its items' flags are up, and combines the batch states in batch order.
//   * A problem with many partials (a lone long problem split over every
//     CTA), or any deferred problem when a CTA per unit covers all their units
//     at once, takes a whole CTA per unit (a task): warp w folds partials w,
//     w + 9, ..., then the warps' states are combined through shared memory
//     in warp order.
//   * The other deferred problems take one warp per unit, nine units to a
//     task, every lane folding all partials of its unit.

// Grid-wide barrier for a cooperative launch: block 0 adds 2^31 - (G - 1),
// the others add 1, so bit 31 of the word flips once all G blocks arrived and
// its low bits return to their start value (zero in a fresh workspace).  The
// arrival is a release-ordered atomic (it publishes the CTA's partials, which
// the __syncthreads before it orders after every thread's stores) and the
// wait an acquire-ordered poll: ~0.5 us shorter than a fence, a relaxed
// atomic and a sleeping poll.  Bounded: returns false after the time limit.
#ifndef FLINT_BARRIER_RELEASE
#define FLINT_BARRIER_RELEASE 1
#endif
__device__ bool grid_barrier(unsigned int* bar, const Smem& S) {
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned int add = blockIdx.x == 0 ? 0x80000000u - (gridDim.x - 1) : 1u;
#if FLINT_BARRIER_RELEASE
    // the arrival publishes this CTA's writes (release); the CTA's other
    // threads' writes are ordered before it by the __syncthreads above
    unsigned int old;
    asm volatile("atom.add.release.gpu.global.u32 %0, [%1], %2;" : "=r"(old) : "l"(bar), "r"(add) : "memory");
#else
    __threadfence();
    const unsigned int old = atomicAdd(bar, add);
#endif
    const unsigned long long t0 = globaltimer_ns();
    int ok = 1;
    for (int spin = 0;; ++spin) {
      unsigned int cur;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(cur) : "l"(bar) : "memory");
      if ((cur ^ old) & 0x80000000u) break;
      if ((spin & 15) == 15 && globaltimer_ns() - t0 > kWaitLimitNs) {
        ok = 0;
        break;
      }
#if !FLINT_BARRIER_RELEASE
      __nanosleep(20);
#endif
    }
#if !FLINT_BARRIER_RELEASE
    __threadfence();
#endif
    S.flags[2] = ok;
  }
  __syncthreads();
  return S.flags[2] != 0;
}

__device__ __forceinline__ unsigned int ld_acquire_u32(const int32_t* p) {
  unsigned int v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Ready-flag mode: folds the warp's partials s0 + first + k * stride (k = 0,
// 1, ...; < s1) into (m, l, acc) in item order, kMergeBatch loads at a time.
// Lane j watches the flag of the j-th item not folded yet (an acquire load);
// the warp's ballot gives the run of raised flags at the front, and every
// whole batch of it (or the last, short batch) is folded.  Batches start at
// fixed multiples of kMergeBatch, as in fold_chunk, so the sums do not depend
// on the mode or on when flags came up.  False if the wait gave up (some CTA
// aborted, or the time limit ran out); the state is then meaningless.
__device__ __forceinline__ bool fold_chunk_wait(const DecodeParams& P, int s0, int s1, int first, int stride,
                                                int head, int c, int q, unsigned int ready, float& m, float& l,
                                                float4& acc) {
  const int lane = threadIdx.x & 31;
  const int i_first = s0 + first;
  const int n = i_first < s1 ? (s1 - i_first + stride - 1) / stride : 0;
  const unsigned long long t0 = globaltimer_ns();
  int done = 0, spin = 0;
  while (done < n) {
    const int k = done + lane;
    const bool up = k >= n || ld_acquire_u32(P.counters + kItemFlags + i_first + k * stride) == ready;
    const unsigned int mask = __ballot_sync(0xffffffffu, up);
    __syncwarp();  // orders every lane's partial loads below after the lanes' acquires
    int take = min(mask == 0xffffffffu ? 32 : __ffs(~mask) - 1, n - done);
    if (take < n - done) take -= take % kMergeBatch;
    if (take == 0) {
      if (ld_relaxed_u32(P.counters + kAbortWord) == ready) return false;
      if ((++spin & 7) == 0 && globaltimer_ns() - t0 > kWaitLimitNs) return false;
      continue;
    }
    for (int b = 0; b < take; b += kMergeBatch) {
      const int cnt = min(kMergeBatch, take - b);
      const int i0 = i_first + (done + b) * stride;
      float mi[kMergeBatch], li[kMergeBatch];
      float4 vi[kMergeBatch];
#pragma unroll
      for (int j = 0; j < kMergeBatch; ++j) {
        const int i = j < cnt ? i0 + j * stride : i0;
        const float* pi = P.partials + static_cast<size_t>(i) * kPartialFloats;
        mi[j] = j < cnt ? __ldcg(pi + kHeads * kDim + head) : -INFINITY;
        li[j] = __ldcg(pi + kHeads * kDim + kHeads + head);
        vi[j] = __ldcg(reinterpret_cast<const float4*>(pi) + partial_f4(head, c, q));
      }
      float mn = m;
#pragma unroll
      for (int j = 0; j < kMergeBatch; ++j) mn = fmaxf(mn, mi[j]);
      const float sa = (m == -INFINITY) ? 0.f : exp2f(m - mn);
      l *= sa;
      acc = make_float4(acc.x * sa, acc.y * sa, acc.z * sa, acc.w * sa);
      m = mn;
#pragma unroll
      for (int j = 0; j < kMergeBatch; ++j) {
        const float sb = (mi[j] == -INFINITY) ? 0.f : exp2f(mi[j] - m);
        l += sb * li[j];
        acc.x += sb * vi[j].x;
        acc.y += sb * vi[j].y;
        acc.z += sb * vi[j].z;
        acc.w += sb * vi[j].w;
      }
    }
    done += take;
  }
  return true;
}

// Grid-barrier mode: Folds partials s0 + first, s0 + first + stride, ... (< s1) into (m, l, acc).
__device__ __forceinline__ void fold_chunk(const DecodeParams& P, int s0, int s1, int first, int stride,
                                           int head, int c, int q, float& m, float& l, float4& acc) {
  for (int i0 = s0 + first; i0 < s1; i0 += kMergeBatch * stride) {
    float mi[kMergeBatch], li[kMergeBatch];
    float4 vi[kMergeBatch];
#pragma unroll
    for (int j = 0; j < kMergeBatch; ++j) {
      const int ij = i0 + j * stride;
      const int i = ij < s1 ? ij : i0;
      const float* pi = P.partials + static_cast<size_t>(i) * kPartialFloats;
      mi[j] = ij < s1 ? __ldcg(pi + kHeads * kDim + head) : -INFINITY;
      li[j] = __ldcg(pi + kHeads * kDim + kHeads + head);
      vi[j] = __ldcg(reinterpret_cast<const float4*>(pi) + partial_f4(head, c, q));
    }
    float mn = m;
#pragma unroll
    for (int j = 0; j < kMergeBatch; ++j) mn = fmaxf(mn, mi[j]);
    const float sa = (m == -INFINITY) ? 0.f : exp2f(m - mn);
    l *= sa;
    acc = make_float4(acc.x * sa, acc.y * sa, acc.z * sa, acc.w * sa);
    m = mn;
#pragma unroll
    for (int j = 0; j < kMergeBatch; ++j) {
      const float sb = (mi[j] == -INFINITY) ? 0.f : exp2f(mi[j] - m);
      l += sb * li[j];
      acc.x += sb * vi[j].x;
      acc.y += sb * vi[j].y;
      acc.z += sb * vi[j].z;
      acc.w += sb * vi[j].w;
    }
  }
}

// Writes values 4q..4q+3 of (head, c), with the sink folded in as finish_head does.
__device__ __forceinline__ void write_chunk(const Problem& pb, int head, int c, int q, float m, float l,
                                            float4 acc, float sink) {
  if (pb.partial) {
    float* o = pb.out + head * kDim + 16 * q;
    const int d0 = dim_d0(c, pb.fp8 != 0), d2 = dim_d2(c, pb.fp8 != 0);
    *reinterpret_cast<float2*>(o + d0) = make_float2(acc.x, acc.y);
    *reinterpret_cast<float2*>(o + d2) = make_float2(acc.z, acc.w);
    if (c == 0 && q == 0) {
      pb.out[kHeads * kDim + head] = m;
      pb.out[kHeads * kDim + kHeads + head] = l;
    }
    return;
  }
  const float scale = sink_scale(m, l, sink);
  float* o = pb.out + head * kDim + 16 * q;
  const int d0 = dim_d0(c, pb.fp8 != 0), d2 = dim_d2(c, pb.fp8 != 0);
  *reinterpret_cast<float2*>(o + d0) = make_float2(acc.x * scale, acc.y * scale);
  *reinterpret_cast<float2*>(o + d2) = make_float2(acc.z * scale, acc.w * scale);
}

// Grid-barrier mode: the merge of the deferred problems by the whole grid
// after the grid barrier; CTA b takes the units of task b (its warps one
// regular unit each, or the whole CTA a wide unit), b + G, ...
__device__ void grid_merge(const DecodeParams& P, const Smem& S) {
  constexpr int kWarps = kThreads / 32;
  constexpr int kUnits = kKvHeads * 8;  // units per problem
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int c = lane & 3;
  {
    const int units = (P.n_deferred - P.n_wide) * kUnits;
    for (int u = blockIdx.x * kWarps + warp; u < units; u += gridDim.x * kWarps) {
      const int p = P.deferred[P.n_wide + u / kUnits];
      const int kvh = (u / 8) % kKvHeads, q = u % 8;
      const int head = kvh * kGroup + (lane >> 2);
      const Problem& pb = P.prob[p];
      const float sink = pb.sinks ? pb.sinks[head] : 0.f;  // in flight with the partials
      float m = -INFINITY, l = 0.f;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      fold_chunk(P, P.seg_item_begin[p], P.seg_item_begin[p + 1], 0, 1, head, c, q, m, l, acc);
      write_chunk(pb, head, c, q, m, l, acc, sink);
    }
  }
  float* red = S.xch;  // [kWarps][32][6] (the hand-over area is free now)
  const int units = P.n_wide * kUnits;
  for (int u = blockIdx.x; u < units; u += gridDim.x) {
    const int p = P.deferred[u / kUnits];
    const int kvh = (u / 8) % kKvHeads, q = u % 8;
    const int head = kvh * kGroup + (lane >> 2);
    const Problem& pb = P.prob[p];
    const float sink = pb.sinks ? pb.sinks[head] : 0.f;
    float m = -INFINITY, l = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    const int s0 = P.seg_item_begin[p], s1 = P.seg_item_begin[p + 1];
#ifdef FLINT_TRACE
    if (threadIdx.x == 0) FLINT_TRACE_SET(13, globaltimer_ns() + 0ull * (s0 + s1 + sink));
#endif
    fold_chunk(P, s0, s1, warp, kWarps, head, c, q, m, l, acc);
#ifdef FLINT_TRACE
    if (threadIdx.x == 0) FLINT_TRACE_SET(14, globaltimer_ns() + 0ull * static_cast<unsigned long long>(acc.x + m + l));
#endif
    float* mine = red + (warp * 32 + lane) * 6;
    mine[0] = m;
    mine[1] = l;
    mine[2] = acc.x;
    mine[3] = acc.y;
    mine[4] = acc.z;
    mine[5] = acc.w;
    __syncthreads();
    if (warp == 0) {
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) M = fmaxf(M, red[(w * 32 + lane) * 6]);
      float L = 0.f;
      float4 A = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float* o = red + (w * 32 + lane) * 6;
        const float sc = (o[0] == -INFINITY) ? 0.f : exp2f(o[0] - M);
        L += sc * o[1];
        A.x += sc * o[2];
        A.y += sc * o[3];
        A.z += sc * o[4];
        A.w += sc * o[5];
      }
      write_chunk(pb, head, c, q, M, L, A, sink);
    }
    if (threadIdx.x == 0) FLINT_TRACE_MARK(15);
    __syncthreads();  // red is reused by the next unit
  }
}

// Ready-flag mode: the launch's end for a CTA whose streaming is over: its
// ticket, then its merge tasks.  A wait that gives up records
// FLINT_ERR_TIMEOUT; the task's output is then left unwritten.
__device__ void merge_tail(const DecodeParams& P, const Smem& S) {
  constexpr int kWarps = kThreads / 32;
  constexpr int kUnits = kKvHeads * 8;  // units per problem
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int c = lane & 3;
  if (t == 0) {
    unsigned int r;
    const int k = take_ticket(P, &r);
    if (S.flags[0]) st_release_u32(P.counters + kAbortWord, r);
    if (k == static_cast<int>(gridDim.x) - 1) P.counters[kQueueHead] = 0;  // ready for the next call
    S.flags[2] = k;
    S.flags[6] = static_cast<int>(r);
    FLINT_TRACE_MARK(8);
  }
  __syncthreads();
  const int rank = S.flags[2];
  const unsigned int ready = static_cast<unsigned int>(S.flags[6]);
  if (rank == static_cast<int>(gridDim.x) - 1) {
    // zero the flags this launch did not raise (no merging CTA reads them)
    for (int i = t; i < kMaxItems; i += kThreads)
      if (!((P.raised[i / 32] >> (i % 32)) & 1u)) P.counters[kItemFlags + i] = 0;
  }
  const int wide_tasks = P.n_wide * kUnits;
  const int units = (P.n_deferred - P.n_wide) * kUnits;
  const int n_tasks = wide_tasks + (units + kWarps - 1) / kWarps;
  float* red = S.xch;  // [kWarps][32][6] (the hand-over area is free now)
  for (int task = rank; task < n_tasks; task += gridDim.x) {
    if (task >= wide_tasks) {
      const int u = (task - wide_tasks) * kWarps + warp;
      if (u < units) {
        const int p = P.deferred[P.n_wide + u / kUnits];
        const int kvh = (u / 8) % kKvHeads, q = u % 8;
        const int head = kvh * kGroup + (lane >> 2);
        const Problem& pb = P.prob[p];
        const float sink = pb.sinks ? pb.sinks[head] : 0.f;  // in flight with the partials
        float m = -INFINITY, l = 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (threadIdx.x == 0) FLINT_TRACE_MARK(13);
        if (fold_chunk_wait(P, P.seg_item_begin[p], P.seg_item_begin[p + 1], 0, 1, head, c, q, ready, m, l,
                            acc))
          write_chunk(pb, head, c, q, m, l, acc, sink);
        else if (lane == 0)
          report_error(P.dev_err, FLINT_ERR_TIMEOUT);
        if (threadIdx.x == 0) FLINT_TRACE_MARK(15);
      }
      continue;
    }
    const int p = P.deferred[task / kUnits];
    const int kvh = (task / 8) % kKvHeads, q = task % 8;
    const int head = kvh * kGroup + (lane >> 2);
    const Problem& pb = P.prob[p];
    const float sink = pb.sinks ? pb.sinks[head] : 0.f;
    float m = -INFINITY, l = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    const int s0 = P.seg_item_begin[p], s1 = P.seg_item_begin[p + 1];
#ifdef FLINT_TRACE
    if (threadIdx.x == 0) FLINT_TRACE_SET(13, globaltimer_ns() + 0ull * (s0 + s1 + sink));
#endif
    const bool ok = fold_chunk_wait(P, s0, s1, warp, kWarps, head, c, q, ready, m, l, acc);
#ifdef FLINT_TRACE
    if (threadIdx.x == 0) FLINT_TRACE_SET(14, globaltimer_ns() + 0ull * static_cast<unsigned long long>(acc.x + m + l));
#endif
    float* mine = red + (warp * 32 + lane) * 6;
    mine[0] = m;
    mine[1] = l;
    mine[2] = acc.x;
    mine[3] = acc.y;
    mine[4] = acc.z;
    mine[5] = acc.w;
    const bool failed = __syncthreads_or(!ok);
    if (warp == 0 && !failed) {
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) M = fmaxf(M, red[(w * 32 + lane) * 6]);
      float L = 0.f;
      float4 A = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float* o = red + (w * 32 + lane) * 6;
        const float sc = (o[0] == -INFINITY) ? 0.f : exp2f(o[0] - M);
        L += sc * o[1];
        A.x += sc * o[2];
        A.y += sc * o[3];
        A.z += sc * o[4];
        A.w += sc * o[5];
      }
      write_chunk(pb, head, c, q, M, L, A, sink);
    }
    if (threadIdx.x == 0) {
      if (failed) report_error(P.dev_err, FLINT_ERR_TIMEOUT);
      FLINT_TRACE_MARK(15);
    }
    __syncthreads();  // red is reused by the next task
  }
}

// kFlags: the launch merges its deferred problems in ready-flag mode
// (P.merge_flags), else after the grid barrier.
template <bool kFlags>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const __grid_constant__ DecodeParams P) {
  // A launch that follows this one in the stream with programmatic
  // dependence may be scheduled from now on (it waits for this grid's
  // completion before it touches global memory, see below).
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
#ifdef FLINT_TRACE
  if (threadIdx.x == 0) {
    unsigned int smid;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
    FLINT_TRACE_MARK(0);
    FLINT_TRACE_SET(10, smid);
  }
#endif
  extern __shared__ uint8_t smem_raw[];
  const Smem S = carve(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int c0 = P.cta_item_begin[blockIdx.x], c1 = P.cta_item_begin[blockIdx.x + 1];
  bool claim = true;
  if (!FLINT_CHECK(P.dev_err, 0 <= c0 && c0 <= c1 && c1 <= P.queue_begin && P.queue_begin + P.n_queue <= P.n_items,
                   1, c0, c1, P.n_items)) {
    c1 = c0;
    claim = false;
  }
  const int smem_end = static_cast<int>(smem_u32(S.in + kInBytes) - smem_u32(smem_raw));
  if (!FLINT_CHECK(P.dev_err, smem_end <= P.smem_bytes, 2, smem_end, P.smem_bytes, 0)) {
    c1 = c0;
    claim = false;
  }
  (void)smem_end;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&S.full[s]), 1);
      mbar_init(smem_u32(&S.empty[s]), kConsumerWarps);
    }
    mbar_init(smem_u32(S.in_full), 1);
    mbar_init(smem_u32(S.in_empty), kConsumerWarps);
    for (int f = 0; f < 8; ++f) S.flags[f] = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (P.prep && threadIdx.x < kDim / 2) S.cs[threadIdx.x] = P.rope_cs[threadIdx.x];
#if FLINT_PREFETCH_MAPS
  if (warp == kConsumerWarps) {
    // the tensor maps are read by TMA from parameter memory: fetch their lines
    // now, while the plan is still being read, not at the first load
    const int n_maps = P.prep ? 2 * P.n_problems : 2;
    for (int i = lane; i < n_maps; i += 32) prefetch_tensormap(&P.maps[i]);
  }
#endif
  __syncthreads();
  // Programmatic dependent launch: everything above overlapped the previous
  // kernel of the stream; wait for it to complete (and its memory to be
  // visible) before any access to the workspace, the caches or the inputs.
  if (P.pdl) asm volatile("griddepcontrol.wait;" ::: "memory");
  if (threadIdx.x == 0) FLINT_TRACE_MARK(1);

  ProducerCount pc{0, 0};
  if (warp == kConsumerWarps) {
    pc = run_producer(P, S, c0, c1, claim, lane);
    if (lane == 0) {
      FLINT_TRACE_MARK(6);
      FLINT_TRACE_SET(11, pc.staged);
    }
  } else {
    run_consumer<kFlags>(P, S, warp, lane);
  }
  __syncthreads();
  if (threadIdx.x == 0) FLINT_TRACE_MARK(7);
  // After an abort, let every issued copy land before the CTA's shared memory
  // goes away (bounded as well; a normal run returns at once).  Only the last
  // armed input phase can still have copies in flight: the producer arms the
  // next one only after the consumers saw this one complete.
  if (warp == kConsumerWarps && lane == 0) {
    if (pc.staged > 0) {
      const unsigned long long t0 = globaltimer_ns();
      while (!mbar_try_wait(smem_u32(S.in_full), static_cast<uint32_t>(pc.staged - 1) & 1u)) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) break;
      }
    }
    const int first = pc.issued > kStages ? pc.issued - kStages : 0;
    for (int s = first; s < pc.issued; ++s) {
      const unsigned long long t0 = globaltimer_ns();
      while (!mbar_try_wait(smem_u32(&S.full[s % kStages]), static_cast<uint32_t>(s / kStages) & 1u)) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) break;
      }
    }
  }
  if (P.grid_merge) {
    if constexpr (kFlags) {
      merge_tail(P, S);
#ifdef FLINT_TRACE
      if (threadIdx.x == 0) FLINT_TRACE_MARK(9);
#endif
    } else if (grid_barrier(reinterpret_cast<unsigned int*>(P.counters + kBarrierWord), S)) {
      // every CTA has made its last claim: ready the queue for the next call
      if (blockIdx.x == 0 && threadIdx.x == 0) P.counters[kQueueHead] = 0;
      if (threadIdx.x == 0) FLINT_TRACE_MARK(8);
      grid_merge(P, S);
#ifdef FLINT_TRACE
      __syncthreads();
      if (threadIdx.x == 0) FLINT_TRACE_MARK(9);
#endif
    } else if (threadIdx.x == 0) {
      report_error(P.dev_err, FLINT_ERR_TIMEOUT);
    }
  }
}

}  // namespace

size_t decode_smem_bytes() {
  return 1024 + static_cast<size_t>(kStages) * kStageBytes + 2 * kStages * sizeof(uint64_t) +
         2 * sizeof(uint64_t) + 64 * sizeof(float2) + 8 * sizeof(int) + kXchSize * sizeof(float) +
         kInBytes;
}

#ifdef FLINT_TRACE
// Copies the trace table (kMaxCtas x kTraceSlots uint64) to host memory.
extern "C" int flint_trace_read(unsigned long long* host) {
  return static_cast<int>(cudaMemcpyFromSymbol(host, g_trace, sizeof(g_trace)));
}
extern "C" int flint_trace_clear() {
  static unsigned long long zero[kMaxCtas][kTraceSlots];
  return static_cast<int>(cudaMemcpyToSymbol(g_trace, zero, sizeof(zero)));
}
#endif

#ifdef FLINT_TEST_HOOKS
// Test builds only: CTA `block` leaves the stage of its tile number `seq`
// (counted over its whole run) unarmed; block = -1 turns the hook off.
extern "C" int flint_test_stall_decode(int block, int seq) {
  const int v[2] = {block, seq};
  return static_cast<int>(cudaMemcpyToSymbol(g_stall_decode, v, sizeof v));
}
#endif

cudaError_t launch_decode(const DecodeParams& p, int grid, cudaStream_t stream) {
  static ContextSet configured[2];
  const int mode = p.merge_flags ? 1 : 0;
  const void* kernel = mode ? reinterpret_cast<const void*>(decode_kernel<true>)
                            : reinterpret_cast<const void*>(decode_kernel<false>);
  cudaError_t e = configure_once(configured[mode], kernel, static_cast<int>(decode_smem_bytes()));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = decode_smem_bytes();
  cfg.stream = stream;
  cudaLaunchAttribute attrs[2];
  int n = 0;
  if (p.grid_merge) {  // the merging CTAs wait for the others: every CTA resident at once
    attrs[n].id = cudaLaunchAttributeCooperative;
    attrs[n].val.cooperative = 1;
    ++n;
  }
  if (p.pdl) {
    attrs[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cfg.attrs = attrs;
  cfg.numAttrs = n;
  e = mode ? cudaLaunchKernelEx(&cfg, decode_kernel<true>, p) : cudaLaunchKernelEx(&cfg, decode_kernel<false>, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace flint
