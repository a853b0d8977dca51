// flint_prefill_prep.cu -- the prefill's per-token pass over a prompt:
// per-head Q/K RMSNorm (+RoPE on the sliding-window layers), q and k rounded
// once to bf16, v converted to fp16 for the attention's P.V product, and the
// cache write ("Day-0 Support for Flint on vLLM", newruntime.com, "What
// happened": fused normalization, rotary-position and cache operations over
// the 8,192-token prefill; hnkhoi.com "Model architecture": per-head Q/K
// RMSNorm, RoPE on the sliding-window layers, NoPE on the full layers).
//
// The pass reads ~10 KB and writes ~12 KB per token and does little
// arithmetic per byte, so it is bound by HBM once enough bytes are in flight.
// A persistent CTA owns a contiguous range of tokens and streams them through
// a ring of shared-memory slots:
//   * warp 8 (producer): one lane issues a token's raw q, k and v rows as three
//     1-D bulk copies (8 KB, 1 KB, 1 KB) into a free slot; while they land,
//     the warp's 32 lanes form the token's 64 (cos, sin) pairs in double
//     precision and its cache row, then arrive on the slot's full barrier
//     (count 32 + the copies' bytes);
//   * warps 0-7 (consumers): the token's 40 rows (32 q, 4 k, 4 v heads) go to
//     16 half-warps, 8 dims per lane (dims 4l..4l+3 and 64+4l..64+4l+3, so
//     RoPE's pairs (i, i+64) stay in one lane); the start rotates by 8
//     half-warps from token to token so the 3-row and 2-row shares alternate.
//     Each consumer lane releases the slot on its empty barrier (count 256)
//     once it has read its rows; the warps never wait for one another.
// Every wait is bounded: a wait that runs out reports FLINT_ERR_TIMEOUT and
// the CTA stops, after letting the copies it issued land.
#include <algorithm>

#include "flint_device.cuh"

namespace flint {

namespace {

#ifndef FLINT_PP_SLOTS
#define FLINT_PP_SLOTS 6
#endif
#ifndef FLINT_PP_CTAS_PER_SM
#define FLINT_PP_CTAS_PER_SM 3
#endif
constexpr int kPpSlots = FLINT_PP_SLOTS;
constexpr int kPpCtasPerSm = FLINT_PP_CTAS_PER_SM;
constexpr int kPpConsumerWarps = 8;
constexpr int kPpProducerWarp = kPpConsumerWarps;
constexpr int kPpThreads = (kPpConsumerWarps + 1) * 32;
constexpr int kPpHalfWarps = 2 * kPpConsumerWarps;               // 16
constexpr int kPpTasks = kHeads + 2 * kKvHeads;                   // 40 rows a token
constexpr int kPpRowBytes = kDim * 2;                             // 256
constexpr uint32_t kPpQBytes = kHeads * kPpRowBytes;              // 8 KiB
constexpr uint32_t kPpKvBytes = kKvHeads * kPpRowBytes;           // 1 KiB
constexpr uint32_t kPpSlotBytes = kPpQBytes + 2 * kPpKvBytes;     // q | k | v: row j at j * 256
static_assert(kPpSlotBytes % 16 == 0, "bulk copies need 16-byte multiples");

struct PpShared {
  uint8_t slot[kPpSlots][kPpSlotBytes];
  // cos, sin and -sin of the slot's token's angles, i < 64
  float cs[kPpSlots][3][kDim / 2];
  long long row[kPpSlots];         // the token's cache row (elements), or -1
  uint64_t full[kPpSlots];
  uint64_t empty[kPpSlots];
  int abort;
};
constexpr size_t kPpSmem = sizeof(PpShared);

#ifdef FLINT_TEST_HOOKS
// {block, token index within the block}: that CTA's producer leaves that
// token's slot unarmed, so the consumers' waits on it run out; {-1, -1} = off.
__device__ int g_stall_prefill_prep[2] = {-1, -1};
#endif

__device__ __forceinline__ bool pp_aborted(const PpShared* S) {
  return *reinterpret_cast<const volatile int*>(&S->abort) != 0;
}

__device__ __forceinline__ void pp_raise_abort(const PrepParams& p, PpShared* S) {
  if (!pp_aborted(S)) report_error(p.dev_err, FLINT_ERR_TIMEOUT);
  *reinterpret_cast<volatile int*>(&S->abort) = 1;
}

// Raise a barrier's expected transaction count without arriving.
__device__ __forceinline__ void mbar_expect_tx_only(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t x) { return make_float2(bf16_lo(x), bf16_hi(x)); }

// The element offset of token t's row (KV head 0) in the cache, or -1 if the
// token is not cached (no cache, or a ring's older tokens).
__device__ long long cache_row_of(const PrepParams& p, int t) {
  if (!p.k_rows) return -1;
  if (p.layout == FLINT_KV_RING && t < p.n_tokens - p.capacity) return -1;
  if (p.layout == FLINT_KV_PAGED) {
    const int blk = p.table[t / kBlock];
    if (blk < 0 || blk >= p.num_blocks) {
      report_error(p.dev_err, FLINT_ERR_INVALID_ARG);
      return -1;
    }
    return (static_cast<long long>(blk) * kBlock + t % kBlock) * kKvHeads * kDim;
  }
  const int slot = p.layout == FLINT_KV_RING ? t % p.capacity : t;
  return static_cast<long long>(slot) * kKvHeads * kDim;
}

// The token's angles for this lane's RoPE pairs: i = 4l + e, e < 4, as
// (cos, sin, -sin) pairs over e = (0, 1) and (2, 3).
struct Turn {
  float2 c[2], s[2], ns[2];
};

// Per-head RMSNorm (+RoPE) of one 128-wide row held by a half-warp: lane l
// (0..15) holds dims 4l..4l+3 (xa) and 64+4l..67+4l (xb) as bf16 pairs, and
// returns them in y[0..1] and y[2..3] (float2 pairs).  y = x * w / sqrt(mean(x^2)
// + eps), then each pair (i, i+64) turns by the token's angle for i.
template <bool kRope>
__device__ __forceinline__ void norm_rope_half(uint2 xa, uint2 xb, const float2 (&w)[4], float eps,
                                               const Turn& tr, float2 (&y)[4]) {
  y[0] = bf16x2_to_float2(xa.x);
  y[1] = bf16x2_to_float2(xa.y);
  y[2] = bf16x2_to_float2(xb.x);
  y[3] = bf16x2_to_float2(xb.y);
  float2 acc = mul2(y[0], y[0]);
  acc = fma2(y[1], y[1], acc);
  acc = fma2(y[2], y[2], acc);
  acc = fma2(y[3], y[3], acc);
  float ss = acc.x + acc.y;
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);  // within the half
  const float r = rsqrtf(fmaf(ss, 1.0f / kDim, eps));
  const float2 rr = make_float2(r, r);
#pragma unroll
  for (int e = 0; e < 4; ++e) y[e] = mul2(mul2(y[e], rr), w[e]);
  if (kRope) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float2 a = y[e], b = y[2 + e];
      y[e] = fma2(b, tr.ns[e], mul2(a, tr.c[e]));      // a cos - b sin
      y[2 + e] = fma2(a, tr.s[e], mul2(b, tr.c[e]));   // b cos + a sin
    }
  }
}

__device__ __forceinline__ uint2 pack_bf16x4(float2 a, float2 b) {
  return make_uint2(pack_bf16x2(a.x, a.y), pack_bf16x2(b.x, b.y));
}

// Four E4M3 codes of (a, b) / s (nearest even, saturating), first in the low byte.
__device__ __forceinline__ uint32_t e4m3x4_of(float2 a, float2 b, float s) {
  const uint32_t lo = f32x2_to_e4m3x2(__fdiv_rn(a.x, s), __fdiv_rn(a.y, s));
  const uint32_t hi = f32x2_to_e4m3x2(__fdiv_rn(b.x, s), __fdiv_rn(b.y, s));
  return (lo & 0xffffu) | (hi << 16);
}

// bf16 -> fp16 to nearest, saturating at +-65504.
__device__ __forceinline__ uint2 bf16x4_to_f16x4(uint2 x) {
  auto sat = [](float f) { return fminf(fmaxf(f, -65504.f), 65504.f); };
  const __half2 a = __floats2half2_rn(sat(bf16_lo(x.x)), sat(bf16_hi(x.x)));
  const __half2 c = __floats2half2_rn(sat(bf16_lo(x.y)), sat(bf16_hi(x.y)));
  return make_uint2(*reinterpret_cast<const uint32_t*>(&a), *reinterpret_cast<const uint32_t*>(&c));
}

// q head j of token t, its row already in (xa, xb).
template <bool kRope>
__device__ __forceinline__ void q_task(const PrepParams& p, int j, int t, uint2 xa, uint2 xb, const Turn& tr,
                                       const float2 (&wq)[4], int l) {
  float2 y[4];
  norm_rope_half<kRope>(xa, xb, wq, p.eps, tr, y);
  uint16_t* o = p.q_out_bf16 + (static_cast<long long>(t) * kHeads + j) * kDim;
  reinterpret_cast<uint2*>(o)[l] = pack_bf16x4(y[0], y[1]);
  reinterpret_cast<uint2*>(o + 64)[l] = pack_bf16x4(y[2], y[3]);
}

// Row task j (32..39) of token t, its row already in (xa, xb): k head j - 32
// or v head j - 36.  `row`: the token's cache row or -1.
template <bool kRope, bool kFp8>
__device__ __forceinline__ void kv_task(const PrepParams& p, int j, int t, uint2 xa, uint2 xb, const Turn& tr,
                                        long long row, const float2 (&wk)[4], int l) {
  if (j < kHeads + kKvHeads) {
    const int hk = j - kHeads;
    float2 y[4];
    norm_rope_half<kRope>(xa, xb, wk, p.eps, tr, y);
    const uint2 ka = pack_bf16x4(y[0], y[1]), kb = pack_bf16x4(y[2], y[3]);
    if (p.k_out) {
      uint16_t* o = p.k_out + (static_cast<long long>(t) * kKvHeads + hk) * kDim;
      reinterpret_cast<uint2*>(o)[l] = ka;
      reinterpret_cast<uint2*>(o + 64)[l] = kb;
    }
    if (row >= 0) {
      if (!kFp8) {
        uint16_t* o = p.k_rows + row + hk * kDim;
        reinterpret_cast<uint2*>(o)[l] = ka;
        reinterpret_cast<uint2*>(o + 64)[l] = kb;
      } else {
        const float s = p.k_scale[hk];
        uint8_t* o = reinterpret_cast<uint8_t*>(p.k_rows) + row + hk * kDim;
        reinterpret_cast<uint32_t*>(o)[l] = e4m3x4_of(y[0], y[1], s);
        reinterpret_cast<uint32_t*>(o + 64)[l] = e4m3x4_of(y[2], y[3], s);
      }
    }
  } else {
    const int hv = j - kHeads - kKvHeads;
    if (p.v_out_f16) {
      uint16_t* o = p.v_out_f16 + (static_cast<long long>(t) * kKvHeads + hv) * kDim;
      reinterpret_cast<uint2*>(o)[l] = bf16x4_to_f16x4(xa);
      reinterpret_cast<uint2*>(o + 64)[l] = bf16x4_to_f16x4(xb);
    }
    if (row >= 0) {
      if (!kFp8) {
        uint16_t* o = p.v_rows + row + hv * kDim;
        reinterpret_cast<uint2*>(o)[l] = xa;
        reinterpret_cast<uint2*>(o + 64)[l] = xb;
      } else {
        const float s = p.v_scale[hv];
        uint8_t* o = reinterpret_cast<uint8_t*>(p.v_rows) + row + hv * kDim;
        reinterpret_cast<uint32_t*>(o)[l] =
            e4m3x4_of(bf16x2_to_float2(xa.x), bf16x2_to_float2(xa.y), s);
        reinterpret_cast<uint32_t*>(o + 64)[l] =
            e4m3x4_of(bf16x2_to_float2(xb.x), bf16x2_to_float2(xb.y), s);
      }
    }
  }
}

// Token range [t0, t1) of this CTA: the T tokens split as evenly as the grid allows.
__device__ __forceinline__ void token_range(int T, int& t0, int& t1) {
  const long long g = gridDim.x, b = blockIdx.x;
  t0 = static_cast<int>(b * T / g);
  t1 = static_cast<int>((b + 1) * T / g);
}

// Which of a token's rows the call needs: q (q_out), k (k_out or the cache),
// v (v_out or the cache); the slot receives only those.
struct Needs {
  bool q, k, v;
  __device__ explicit Needs(const PrepParams& p)
      : q(p.q_out_bf16 != nullptr), k(p.k_out != nullptr || p.k_rows != nullptr),
        v(p.v_raw != nullptr && (p.v_out_f16 != nullptr || p.k_rows != nullptr)) {}
  __device__ uint32_t bytes() const { return (q ? kPpQBytes : 0u) + (k ? kPpKvBytes : 0u) + (v ? kPpKvBytes : 0u); }
};

// Producer warp.  Returns the number of tokens whose slots it handed out
// (armed or, under the test hook, left unarmed); the drain's bound.
template <bool kRope>
__device__ int run_producer(const PrepParams& p, PpShared* S, int t0, int n, int lane) {
  const Needs need(p);
  const uint32_t bytes = need.bytes();
  // theta^(-2i/128) for this lane's two pairs, i = lane and lane + 32
  const double f0 = kRope ? pow(p.theta, -2.0 * lane / kDim) : 0.0;
  const double f1 = kRope ? pow(p.theta, -2.0 * (lane + 32) / kDim) : 0.0;
  int k = 0;
  for (; k < n; ++k) {
    const int s = k % kPpSlots;
    if (k >= kPpSlots) {
      const bool ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&S->empty[s]),
                                                        static_cast<uint32_t>(k / kPpSlots - 1) & 1u, &S->abort));
      if (!ok) {
        if (lane == 0) pp_raise_abort(p, S);
        break;
      }
    }
    if (__any_sync(0xffffffffu, pp_aborted(S))) break;
    const int t = t0 + k;
#ifdef FLINT_TEST_HOOKS
    if (static_cast<int>(blockIdx.x) == g_stall_prefill_prep[0] && k == g_stall_prefill_prep[1]) continue;
#endif
    const uint32_t full = smem_u32(&S->full[s]);
    if (lane == 0) {
      mbar_expect_tx_only(full, bytes);
      const uint32_t dst = smem_u32(S->slot[s]);
      if (need.q) bulk_copy_g2s(dst, p.q_raw + static_cast<long long>(t) * kHeads * kDim, kPpQBytes, full);
      if (need.k)
        bulk_copy_g2s(dst + kPpQBytes, p.k_raw + static_cast<long long>(t) * kKvHeads * kDim, kPpKvBytes, full);
      if (need.v)
        bulk_copy_g2s(dst + kPpQBytes + kPpKvBytes, p.v_raw + static_cast<long long>(t) * kKvHeads * kDim,
                      kPpKvBytes, full);
      S->row[s] = cache_row_of(p, t);
    }
    if (kRope) {
      // the angle formed and reduced in double precision (a float angle near
      // position 1e5 would be off by ~1e-2 rad), each value rounded once
      double sn, c;
      sincos(static_cast<double>(t) * f0, &sn, &c);
      S->cs[s][0][lane] = static_cast<float>(c);
      S->cs[s][1][lane] = static_cast<float>(sn);
      S->cs[s][2][lane] = -static_cast<float>(sn);
      sincos(static_cast<double>(t) * f1, &sn, &c);
      S->cs[s][0][lane + 32] = static_cast<float>(c);
      S->cs[s][1][lane + 32] = static_cast<float>(sn);
      S->cs[s][2][lane + 32] = -static_cast<float>(sn);
    }
    mbar_arrive(full);  // release: this lane's angles and, for lane 0, the row
  }
  return k;
}

// After an abort: let the copies still in flight land before the CTA's shared
// memory goes away (bounded).  Only the last kPpSlots tokens handed out can be
// pending: a slot is refilled only after its previous token was consumed,
// which needed that token's copies landed.
__device__ void pp_drain(const PpShared* S, int handed_out) {
  const unsigned long long t0 = globaltimer_ns();
  for (int k = max(0, handed_out - kPpSlots); k < handed_out; ++k) {
#ifdef FLINT_TEST_HOOKS
    if (static_cast<int>(blockIdx.x) == g_stall_prefill_prep[0] && k == g_stall_prefill_prep[1]) continue;
#endif
    const uint32_t bar = smem_u32(&S->full[k % kPpSlots]);
    const uint32_t parity = static_cast<uint32_t>(k / kPpSlots) & 1u;
    while (!mbar_try_wait(bar, parity))
      if (globaltimer_ns() - t0 > kWaitLimitNs) return;
  }
}

// Consumer warp: every token of the CTA's range, 2 or 3 of its 40 rows per
// half-warp.
template <bool kRope, bool kFp8>
__device__ void run_consumer(const PrepParams& p, PpShared* S, int t0, int n, int warp, int lane) {
  const Needs need(p);
  const int l = lane & 15;
  const int h = 2 * warp + (lane >> 4);
  float2 wq[4], wk[4];
  {
    const uint2 qa = reinterpret_cast<const uint2*>(p.w_q)[l], qb = reinterpret_cast<const uint2*>(p.w_q + 64)[l];
    const uint2 ka = reinterpret_cast<const uint2*>(p.w_k)[l], kb = reinterpret_cast<const uint2*>(p.w_k + 64)[l];
    wq[0] = bf16x2_to_float2(qa.x);
    wq[1] = bf16x2_to_float2(qa.y);
    wq[2] = bf16x2_to_float2(qb.x);
    wq[3] = bf16x2_to_float2(qb.y);
    wk[0] = bf16x2_to_float2(ka.x);
    wk[1] = bf16x2_to_float2(ka.y);
    wk[2] = bf16x2_to_float2(kb.x);
    wk[3] = bf16x2_to_float2(kb.y);
  }
  for (int k = 0; k < n; ++k) {
    const int s = k % kPpSlots;
    const bool ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&S->full[s]),
                                                      static_cast<uint32_t>(k / kPpSlots) & 1u, &S->abort));
    if (!ok) {
      if (lane == 0) pp_raise_abort(p, S);
      break;
    }
    const int t = t0 + k;
    // rows r, r + 16 (q heads) and, for r < 8, r + 32 (k or v); the two
    // halves of a warp take r and r + 1 (r even), so a warp's third rows are
    // of one kind (the kinds change at rows 32 and 36)
    const int r = (h + (kPpHalfWarps / 2) * (k & 1)) & (kPpHalfWarps - 1);
    const bool third = r + 2 * kPpHalfWarps < kPpTasks;
    // every row this lane needs, read before any result is stored
    const uint8_t* slot = S->slot[s];
    uint2 xa[3], xb[3];
#pragma unroll
    for (int u = 0; u < 3; ++u) {
      const int j = r + u * kPpHalfWarps;
      if (u < 2 || third) {
        xa[u] = reinterpret_cast<const uint2*>(slot + j * kPpRowBytes)[l];
        xb[u] = reinterpret_cast<const uint2*>(slot + j * kPpRowBytes + 128)[l];
      }
    }
    Turn tr;
    if (kRope) {
      const float4 c = reinterpret_cast<const float4*>(S->cs[s][0])[l];
      const float4 sn = reinterpret_cast<const float4*>(S->cs[s][1])[l];
      const float4 ns = reinterpret_cast<const float4*>(S->cs[s][2])[l];
      tr.c[0] = make_float2(c.x, c.y);
      tr.c[1] = make_float2(c.z, c.w);
      tr.s[0] = make_float2(sn.x, sn.y);
      tr.s[1] = make_float2(sn.z, sn.w);
      tr.ns[0] = make_float2(ns.x, ns.y);
      tr.ns[1] = make_float2(ns.z, ns.w);
    }
    const long long row = S->row[s];
    mbar_arrive(smem_u32(&S->empty[s]));  // this lane's reads are done: release the slot
    if (need.q) {
      q_task<kRope>(p, r, t, xa[0], xb[0], tr, wq, l);
      q_task<kRope>(p, r + kPpHalfWarps, t, xa[1], xb[1], tr, wq, l);
    }
    const int j = r + 2 * kPpHalfWarps;
    if (third && (j < kHeads + kKvHeads ? need.k : need.v)) kv_task<kRope, kFp8>(p, j, t, xa[2], xb[2], tr, row, wk, l);
  }
}

template <bool kRope, bool kFp8>
__global__ void __launch_bounds__(kPpThreads, kPpCtasPerSm) prefill_prep_kernel(const __grid_constant__ PrepParams p) {
  extern __shared__ uint8_t pp_raw[];
  PpShared* S = reinterpret_cast<PpShared*>((reinterpret_cast<uintptr_t>(pp_raw) + 127) & ~uintptr_t(127));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int t0, t1;
  token_range(p.n_tokens, t0, t1);
  const int n = t1 - t0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPpSlots; ++s) {
      mbar_init(smem_u32(&S->full[s]), 32);
      mbar_init(smem_u32(&S->empty[s]), kPpConsumerWarps * 32);
    }
    S->abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncthreads();

  int handed_out = 0;
  if (warp == kPpProducerWarp) {
    handed_out = run_producer<kRope>(p, S, t0, n, lane);
  } else {
    run_consumer<kRope, kFp8>(p, S, t0, n, warp, lane);
  }
  // The consumers leave once they consumed every token (so every copy has
  // landed) or on an abort; after an abort the producer lets its copies land.
  __syncthreads();
  if (warp == kPpProducerWarp && lane == 0 && pp_aborted(S)) pp_drain(S, handed_out);
}

}  // namespace

#ifdef FLINT_TEST_HOOKS
// Test builds only: CTA `block` leaves the slot of its token `k` (counted from
// the start of its range) unarmed; block = -1 turns the hook off.
extern "C" int flint_test_stall_prefill_prep(int block, int k) {
  const int v[2] = {block, k};
  return static_cast<int>(cudaMemcpyToSymbol(g_stall_prefill_prep, v, sizeof v));
}
#endif

int prefill_prep_grid(int T, int num_sms) {
  return static_cast<int>(std::min<long long>(T, static_cast<long long>(kPpCtasPerSm) * num_sms));
}

namespace {

// (internal linkage: a function-local static of a template with external
// linkage is one object across every library loaded in the process, so a
// second build of this library would find its context already configured)
template <bool kRope, bool kFp8>
cudaError_t launch_prefill_prep_t(const PrepParams& p, int grid, cudaStream_t stream) {
  static ContextSet configured;
  const int smem = static_cast<int>(kPpSmem) + 128;
  const void* fn = reinterpret_cast<const void*>(prefill_prep_kernel<kRope, kFp8>);
  cudaError_t e = configure_once(configured, fn, smem);
  if (e != cudaSuccess) return e;
  prefill_prep_kernel<kRope, kFp8><<<grid, kPpThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_prep(const PrepParams& p, int grid, cudaStream_t stream) {
  if (p.apply_rope)
    return p.fp8 ? launch_prefill_prep_t<true, true>(p, grid, stream) : launch_prefill_prep_t<true, false>(p, grid, stream);
  return p.fp8 ? launch_prefill_prep_t<false, true>(p, grid, stream) : launch_prefill_prep_t<false, false>(p, grid, stream);
}

}  // namespace flint
