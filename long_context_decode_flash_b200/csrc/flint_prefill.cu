// flint_prefill.cu -- attention of a prompt over itself (prefill): for every
// query position t of a T-token prompt and every query head h (KV head
// h / 8, learned sink logit), over the keys of positions
// max(0, t - window + 1) .. t (sliding-window layers, window 513) or 0 .. t
// (full layers):
//     out[t][h] = sum_j e^(s_j - M) V[j] / (sum_j e^(s_j - M) + e^(sink_h - M)),
//     s_j = q[t][h] . K[j] / sqrt(128),  M = max(max_j s_j, sink_h)
// ("Day-0 Support for Flint on vLLM", hnkhoi.com, "Model architecture"; the
// 8,192-token prefill of newruntime.com, "What happened").
//
// How (5th-generation tensor cores, tcgen05): the work is split into units
// (block of 16 query tokens, KV head g); a unit's 128 query rows are the 16
// tokens x the 8 heads of the group (row r = 8 * token + head), so every K/V
// tile serves all 8 heads.  The kernel is persistent: one CTA per SM (its 512
// TMEM columns fill the SM) walks its share of the units, dealt longest first
// in rounds of alternating direction; tiles, ring stages and barrier phases
// are counted across the CTA's units.  Ten warps:
//   warp 8     TMA producer: per unit the Q tile (once the previous unit's S
//              MMAs are done with it), then 128-key K and V tiles through 3-
//              and 2-stage rings (128-byte swizzle, two 64-dim boxes a tile).
//   warp 9     allocates the 512 TMEM columns; its lane 0 issues the MMAs:
//              S = Q K^T (bf16, M 128, N 128, K 128) into one of two TMEM S
//              buffers, and O += P V (fp16, K 128) with P read from TMEM and V
//              from shared memory (dims-major operand).
//   warps 0-7  softmax in two warpgroups; thread (wg, r) owns row r (TMEM
//              lane r) and the 64 keys 64 wg .. 64 wg + 63 of every tile, and
//              the 64 output dims 64 wg .. 64 wg + 63.  Per tile: S from TMEM,
//              the causal / window mask on boundary tiles, the row maximum
//              exchanged between the two warpgroups through shared memory, an
//              fp32 online softmax in log2 units whose running maximum moves
//              only when a tile exceeds it by more than 2^8 (then O is
//              rescaled in TMEM), P back to TMEM; at the end of a unit O, the
//              sink and the store through a per-warp staging tile.
// P is rounded to fp16 (P <= 2^8 under the lazy maximum, relative error
// 2^-12) and V arrives in fp16 (exact for bf16 values in the fp16 normal
// range), so one PV product keeps the output within a few 1e-4 of the exact
// attention for unit-scale values.
// TMEM columns: S0 [0,128), S1 [128,256), P [256,320) (fp16 pairs), O
// [384,512).  Every wait is bounded; a timeout raises FLINT_ERR_TIMEOUT.
#include <math.h>

#include <algorithm>

#include "flint_device.cuh"

namespace flint {

namespace {

constexpr int kPq = 16;                    // query tokens per CTA
constexpr int kRows = kPq * kGroup;        // 128 query rows (token, head)
constexpr int kPkv = 128;                  // keys per tile
constexpr int kKs = 3, kVs = 2;            // K and V ring stages
constexpr int kSoftWarps = 8;              // two warpgroups
constexpr int kTmaWarp = 8, kMmaWarp = 9;
constexpr int kPfThreads = 320;
constexpr uint32_t kHalfBytes = kPkv * 128;            // one 64-dim box of a tile: 16 KiB
constexpr uint32_t kTileBytes = 2 * kHalfBytes;        // 32 KiB
constexpr uint32_t kQBytes = 2 * kRows * 128;          // 32 KiB
constexpr uint32_t kOffK = kQBytes;
constexpr uint32_t kOffV = kOffK + kKs * kTileBytes;
constexpr uint32_t kOffRed = kOffV + kVs * kTileBytes;  // row-maximum exchange [2 tiles][2 wg][128]
constexpr uint32_t kOffL = kOffRed + 2 * 2 * kRows * 4;    // row-sum exchange [2 wg][128], once per unit
constexpr uint32_t kOffStage = kOffL + 2 * kRows * 4;  // output staging, [softmax warp][32 rows][16 floats]
constexpr uint32_t kStageWarpBytes = 32 * 16 * 4;
constexpr uint32_t kOffBar = kOffStage + kSoftWarps * kStageWarpBytes;
constexpr size_t kPfSmem = kOffBar + 256 + 1024;        // barriers, TMEM address, flags; alignment slack
constexpr float kPfLog2e = 1.4426950408889634f;
constexpr float kPfScale = static_cast<float>(1.4426950408889634 * 0.08838834764831845);
constexpr float kTau = 8.0f;               // lazy-rescale threshold (log2 units)
constexpr uint32_t kColS = 0, kColP = 256, kColO = 384;

// Instruction descriptors (kind::f16), fp32 D, M 128, N 128.  S: bf16 A and
// B, both K-major.  PV: fp16 A and B, B (V) dims-major.
constexpr uint32_t kIdescS = (1u << 4) | (1u << 7) | (1u << 10) | ((kPkv >> 3) << 17) | ((128 >> 4) << 24);
constexpr uint32_t kIdescPV = (1u << 4) | (1u << 16) | ((kDim >> 3) << 17) | ((128 >> 4) << 24);

struct Bars {  // at kOffBar
  uint64_t q_full;        // the unit's Q tile landed (phase = unit)
  uint64_t q_empty;       // every S MMA of the unit completed: Q may be replaced
  uint64_t k_full[kKs], k_empty[kKs];
  uint64_t v_full[kVs], v_empty[kVs];
  uint64_t s_full[2];
  uint64_t p_full;
  uint64_t pv_done;
  uint64_t mma_done;
  uint64_t red_full[2];   // both softmax warpgroups wrote their row maxima (per tile parity)
  uint64_t l_full;        // ... their row sums (once per unit)
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Bars) <= 256, "barrier block");

// Shared-memory matrix descriptor, 128-byte swizzle (sm_100 version 1).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

__device__ __forceinline__ void umma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void umma_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
// Arrive once on `bar` when every tcgen05 operation this thread issued so far
// has completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

#define FLINT_R8(i) "=r"(r[i]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3]), "=r"(r[i + 4]), \
                    "=r"(r[i + 5]), "=r"(r[i + 6]), "=r"(r[i + 7])
#define FLINT_W8(i) "r"(r[i]), "r"(r[i + 1]), "r"(r[i + 2]), "r"(r[i + 3]), "r"(r[i + 4]), \
                    "r"(r[i + 5]), "r"(r[i + 6]), "r"(r[i + 7])

// 32 consecutive columns of this warp's 32 lanes: lane i gets row i.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : FLINT_R8(0), FLINT_R8(8), FLINT_R8(16), FLINT_R8(24)
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      FLINT_W8(0), FLINT_W8(8), FLINT_W8(16), FLINT_W8(24)
      : "memory");
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x for a pair on the FMA pipe, for x <= 2^8 (the softmax's exponents):
// x = j + f with j = rint(x) (x + 1.5 * 2^23 puts rint(x) in the low bits)
// and f in [-1/2, 1/2]; 2^f is the degree-4 polynomial interpolating 2^f at
// the five Chebyshev nodes of [-1/2, 1/2] (relative error below 3.6e-6 with
// float coefficients); j joins the exponent field by an integer add.  x is
// clamped at -127 so that the add stays in range (results below 2^-126 come
// out as 0 or tiny values, which the fp16 P rounds to 0).
__device__ __forceinline__ float2 ex2_fma2(float2 x) {
  x = make_float2(fmaxf(x.x, -127.0f), fmaxf(x.y, -127.0f));
  const float2 t = add2(x, make_float2(12582912.0f, 12582912.0f));
  const float2 f = fma2(add2(t, make_float2(-12582912.0f, -12582912.0f)), make_float2(-1.0f, -1.0f), x);
  float2 q = fma2(make_float2(0x1.3cbf6p-7f, 0x1.3cbf6p-7f), f, make_float2(0x1.ca1ce2p-5f, 0x1.ca1ce2p-5f));
  q = fma2(q, f, make_float2(0x1.ebfa4cp-3f, 0x1.ebfa4cp-3f));
  q = fma2(q, f, make_float2(0x1.62e0c2p-1f, 0x1.62e0c2p-1f));
  q = fma2(q, f, make_float2(1.0f, 1.0f));
  return make_float2(__int_as_float(__float_as_int(q.x) + (__float_as_int(t.x) << 23)),
                     __int_as_float(__float_as_int(q.y) + (__float_as_int(t.y) << 23)));
}

// Bounded wait shared by all lanes of a warp: true only if every lane saw
// the phase complete.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, Bars* B) {
  const bool ok = mbar_wait(bar, parity, &B->abort);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void raise_abort(const PrefillParams& p, Bars* B) {
  if (!B->abort) report_error(p.dev_err, FLINT_ERR_TIMEOUT);
  B->abort = 1;
}

#ifdef FLINT_TEST_HOOKS
// {block, K tile}: that CTA's producer leaves that K tile unarmed; {-1, -1} = off.
__device__ int g_stall_prefill[2] = {-1, -1};
#endif

// Q, K and V tiles whose loads the producer issued (the drain's bound).
struct Issued {
  int k, v, q;
};

__device__ __forceinline__ bool aborted(const Bars* B) {
  return *reinterpret_cast<const volatile int*>(&B->abort) != 0;
}

struct Work {
  int t0, g, j_first, n;
  __device__ bool interior(int jj, int window) const {
    const int k0 = (j_first + jj) * kPkv;
    const int t_hi = t0 + kPq - 1;
    return k0 + kPkv - 1 <= t0 && (window == 0 || k0 > t_hi - window);
  }
};

// Units (block of 16 query tokens, KV head), numbered longest first.
__device__ __forceinline__ int n_units(const PrefillParams& p) { return (p.T + kPq - 1) / kPq * kKvHeads; }

__device__ __forceinline__ Work work_of_unit(const PrefillParams& p, int u) {
  const int nblk = (p.T + kPq - 1) / kPq;
  const int qb = nblk - 1 - u / kKvHeads;
  Work w;
  w.g = u % kKvHeads;
  w.t0 = qb * kPq;
  const int t_last = min(w.t0 + kPq - 1, p.T - 1);
  w.j_first = p.window > 0 ? max(0, w.t0 - (p.window - 1)) / kPkv : 0;
  w.n = t_last / kPkv - w.j_first + 1;
  return w;
}

// The i-th unit of this CTA: rounds of gridDim.x units, dealt in alternating
// directions so that every CTA's total is close to the mean; >= n_units(p)
// past the CTA's last unit.
__device__ __forceinline__ int unit_of(int i) {
  const int G = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
  return i * G + ((i & 1) ? G - 1 - c : c);
}

// The producer: per unit, the Q tile (once the previous unit's S MMAs are
// done with the buffer), then the unit's K and V tiles through the rings,
// counted across units.  Returns what it issued; once the CTA aborted it
// issues nothing more.
__device__ Issued run_tma(const PrefillParams& p, uint8_t* smem, Bars* B) {
  const uint32_t base = smem_u32(smem);
  Issued n{0, 0, 0};
  const int units = n_units(p);
  int T = 0;  // the CTA's tile count so far
  for (int i = 0;; ++i) {
    const int u = unit_of(i);
    if (u >= units) break;
    const Work w = work_of_unit(p, u);
    if (i > 0 && !mbar_wait(smem_u32(&B->q_empty), static_cast<uint32_t>(i - 1) & 1u, &B->abort)) {
      raise_abort(p, B);
      return n;
    }
    if (aborted(B)) return n;
    mbar_expect_tx(smem_u32(&B->q_full), kQBytes);
    tma_load_4d(base, &p.q_map, smem_u32(&B->q_full), 0, w.g * kGroup, w.t0, 0);
    tma_load_4d(base + kRows * 128, &p.q_map, smem_u32(&B->q_full), 64, w.g * kGroup, w.t0, 0);
    n.q = i + 1;
    for (int jj = 0; jj < w.n; ++jj) {
      const int tt = T + jj;
      const int k0 = (w.j_first + jj) * kPkv;
      const int sk = tt % kKs, sv = tt % kVs;
      if (tt >= kKs && !mbar_wait(smem_u32(&B->k_empty[sk]), static_cast<uint32_t>(tt / kKs - 1) & 1u, &B->abort)) {
        raise_abort(p, B);
        return n;
      }
      if (aborted(B)) return n;
      const uint32_t dk = base + kOffK + sk * kTileBytes;
#ifdef FLINT_TEST_HOOKS
      if (!(static_cast<int>(blockIdx.x) == g_stall_prefill[0] && tt == g_stall_prefill[1]))
#endif
      {
        mbar_expect_tx(smem_u32(&B->k_full[sk]), kTileBytes);
        tma_load_4d(dk, &p.k_map, smem_u32(&B->k_full[sk]), 0, w.g, k0, 0);
        tma_load_4d(dk + kHalfBytes, &p.k_map, smem_u32(&B->k_full[sk]), 64, w.g, k0, 0);
      }
      n.k = tt + 1;
      if (tt >= kVs && !mbar_wait(smem_u32(&B->v_empty[sv]), static_cast<uint32_t>(tt / kVs - 1) & 1u, &B->abort)) {
        raise_abort(p, B);
        return n;
      }
      if (aborted(B)) return n;
      const uint32_t dv = base + kOffV + sv * kTileBytes;
      mbar_expect_tx(smem_u32(&B->v_full[sv]), kTileBytes);
      tma_load_4d(dv, &p.v_map, smem_u32(&B->v_full[sv]), 0, w.g, k0, 0);
      tma_load_4d(dv + kHalfBytes, &p.v_map, smem_u32(&B->v_full[sv]), 64, w.g, k0, 0);
      n.v = tt + 1;
    }
    T += w.n;
  }
  return n;
}

// After an abort: let the copies still in flight land before the CTA's shared
// memory goes away (bounded).  Only the last kKs K and kVs V tiles the
// producer issued can be pending: it issues tile j into a stage only after the
// stage's tile j - kKs (or j - kVs) was consumed, which needed it landed.  The
// waits must be on those issued phases: a parity wait on a later, never armed
// phase of the same stage would pass on an older one while a copy still lands.
__device__ void drain_tma(Issued n, Bars* B) {
  const unsigned long long t0 = globaltimer_ns();
  auto wait = [&](uint32_t bar, uint32_t parity) {
    while (!mbar_try_wait(bar, parity))
      if (globaltimer_ns() - t0 > kWaitLimitNs) return;
  };
  if (n.q > 0) wait(smem_u32(&B->q_full), static_cast<uint32_t>(n.q - 1) & 1u);
  for (int jj = max(0, n.k - kKs); jj < n.k; ++jj)
    wait(smem_u32(&B->k_full[jj % kKs]), static_cast<uint32_t>(jj / kKs) & 1u);
  for (int jj = max(0, n.v - kVs); jj < n.v; ++jj)
    wait(smem_u32(&B->v_full[jj % kVs]), static_cast<uint32_t>(jj / kVs) & 1u);
}

// S[jj & 1] = Q K_jj^T for the CTA's tile jj: 8 MMAs of K = 16 dims (32 bytes
// inside a swizzled 128-byte row; the second 64 dims in the second box).
// last: the unit's last S, after which Q may be replaced.
__device__ __forceinline__ bool issue_s(const PrefillParams& p, int jj, bool last, uint32_t base, uint32_t tmem,
                                        Bars* B) {
  const int sk = jj % kKs;
  if (!mbar_wait(smem_u32(&B->k_full[sk]), static_cast<uint32_t>(jj / kKs) & 1u, &B->abort)) return false;
  tc_fence_after();
  const uint32_t qa = base, kb = base + kOffK + sk * kTileBytes;
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint32_t off = (kk >> 2) * (kRows * 128) + (kk & 3) * 32;
    const uint32_t offk = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
    umma_ss(tmem + kColS + (jj & 1) * kPkv, sw128_desc(qa + off, 16, 1024), sw128_desc(kb + offk, 16, 1024),
            kIdescS, kk > 0 ? 1u : 0u);
  }
  umma_commit(smem_u32(&B->k_empty[sk]));
  umma_commit(smem_u32(&B->s_full[jj & 1]));
  if (last) umma_commit(smem_u32(&B->q_empty));
  return true;
}

// The MMA thread, over the CTA's units with its tiles counted across them.
// Per unit: S of the first two tiles, then per tile PV and the S two tiles
// ahead within the unit.  The first PV of a unit overwrites O: every softmax
// warp read the previous unit's O out of TMEM before it wrote its half of
// this tile's P, so p_full already orders that PV after the reads.  The next unit's first S come after
// this unit's last PV, so that no PV waits for the next Q tile.
__device__ void run_mma(const PrefillParams& p, uint32_t base, uint32_t tmem, Bars* B) {
  const int units = n_units(p);
  int T = 0;
  Work w = work_of_unit(p, unit_of(0));
  bool ok = mbar_wait(smem_u32(&B->q_full), 0, &B->abort);
  if (ok) ok = issue_s(p, 0, w.n == 1, base, tmem, B);
  if (ok && w.n > 1) ok = issue_s(p, 1, w.n == 2, base, tmem, B);
  for (int i = 0; ok; ++i) {
    for (int jj = 0; ok && jj < w.n; ++jj) {
      const int tt = T + jj;
      const int sv = tt % kVs;
      ok = mbar_wait(smem_u32(&B->p_full), static_cast<uint32_t>(tt) & 1u, &B->abort) &&
           mbar_wait(smem_u32(&B->v_full[sv]), static_cast<uint32_t>(tt / kVs) & 1u, &B->abort);
      if (!ok) break;
      tc_fence_after();
      const uint32_t vb = base + kOffV + sv * kTileBytes;
      // O += P V: K = 16 keys per MMA (rows 16kk.. of both 64-dim boxes; the
      // fp16 pairs of keys 16kk .. 16kk + 15 are columns 8kk .. 8kk + 7 of P)
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        umma_ts(tmem + kColO, tmem + kColP + kk * 8, sw128_desc(vb + kk * 16 * 128, kHalfBytes, 1024), kIdescPV,
                (jj > 0 || kk > 0) ? 1u : 0u);
      umma_commit(smem_u32(&B->v_empty[sv]));
      umma_commit(smem_u32(&B->pv_done));
      if (jj + 2 < w.n) ok = issue_s(p, tt + 2, jj + 2 == w.n - 1, base, tmem, B);
    }
    if (!ok) break;
    T += w.n;
    const int u = unit_of(i + 1);
    if (u >= units) break;
    w = work_of_unit(p, u);
    ok = mbar_wait(smem_u32(&B->q_full), static_cast<uint32_t>(i + 1) & 1u, &B->abort);
    if (ok) ok = issue_s(p, T, w.n == 1, base, tmem, B);
    if (ok && w.n > 1) ok = issue_s(p, T + 1, w.n == 2, base, tmem, B);
  }
  if (!ok) raise_abort(p, B);
  // let every issued MMA finish before the CTA ends (its TMEM is freed)
  umma_commit(smem_u32(&B->mma_done));
  const unsigned long long t0 = globaltimer_ns();
  while (!mbar_try_wait(smem_u32(&B->mma_done), 0)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) break;
  }
}

// One unit (the CTA's i-th; its tiles are the CTA's T .. T + w.n - 1).
// Returns false if a wait ran out (the caller stops).
__device__ bool softmax_unit(const PrefillParams& p, const Work& w, int i, int T, uint32_t tmem, uint8_t* smem,
                             Bars* B, int warp, int lane) {
  const int wg = warp >> 2;               // key half of every tile, dims half of O
  const int r = (warp & 3) * 32 + lane;   // TMEM lane = query row
  const int t = w.t0 + (r >> 3);          // its token
  const int h = w.g * kGroup + (r & 7);   // its query head
  const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
  float* red = reinterpret_cast<float*>(smem + kOffRed);  // [tile parity][wg][row]
  float m = -INFINITY, l = 0.f;           // m in log2 units
  bool ok = true;
  constexpr int kH = kPkv / 2;            // keys of this thread per tile
  for (int jj = 0; jj < w.n; ++jj) {
    const int tt = T + jj;  // the CTA's tile count: buffers and barrier phases
    if (!warp_wait(smem_u32(&B->s_full[tt & 1]), static_cast<uint32_t>(tt >> 1) & 1u, B)) {
      ok = false;
      break;
    }
    tc_fence_after();
    static_assert(kH == 64, "two 32-column loads per tile");
    float s[kH];  // raw scores q.k
    {
      uint32_t v0[32], v1[32];
      tmem_ld32(lane_base + kColS + (tt & 1) * kPkv + kH * wg, v0);
      tmem_ld32(lane_base + kColS + (tt & 1) * kPkv + kH * wg + 32, v1);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        s[i] = __uint_as_float(v0[i]);
        s[32 + i] = __uint_as_float(v1[i]);
      }
    }
    if (!w.interior(jj, p.window)) {
      const int k0 = (w.j_first + jj) * kPkv + kH * wg;
#pragma unroll
      for (int i = 0; i < kH; ++i) {
        const int key = k0 + i;
        if (key > t || (p.window > 0 && key <= t - p.window)) s[i] = -INFINITY;
      }
    }
    float mq[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) mq[q] = s[q];
#pragma unroll
    for (int i = 8; i < kH; i += 2) mq[(i >> 1) & 7] = max3(mq[(i >> 1) & 7], s[i], s[i + 1]);
    const float mh = max3(max3(mq[0], mq[1], mq[2]), max3(mq[3], mq[4], mq[5]), fmaxf(mq[6], mq[7]));
    // exchange the half-row maxima (every thread arrives; bounded wait)
    float* slot = red + (tt & 1) * 2 * kRows;
    slot[wg * kRows + r] = mh;
    mbar_arrive(smem_u32(&B->red_full[tt & 1]));
    if (!warp_wait(smem_u32(&B->red_full[tt & 1]), static_cast<uint32_t>(tt >> 1) & 1u, B)) {
      ok = false;
      break;
    }
    const float mx = fmaxf(slot[r], slot[kRows + r]) * kPfScale;  // the row's tile maximum, log2 units
    const bool need = mx > m + kTau || (m == -INFINITY && mx > -INFINITY);
    float factor = 1.f;
    if (need) {
      factor = (m == -INFINITY) ? 0.f : ex2(m - mx);
      m = mx;
      l *= factor;
    }
    const float mu = (m == -INFINITY) ? 0.f : m;
    uint32_t pk[kH / 2];  // fp16 pairs
    // scale, shift and sum a pair of scores per paired-fp32 instruction
    const float2 scale2 = make_float2(kPfScale, kPfScale), nmu2 = make_float2(-mu, -mu);
    float2 ls[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
    for (int c = 0; c < kH / 2; ++c) {
      const float2 x = fma2(make_float2(s[2 * c], s[2 * c + 1]), scale2, nmu2);
      // one pair in four on the FMA pipe: the MUFU unit bounds this loop
      const float2 pp = (c & 3) == 3 ? ex2_fma2(x) : make_float2(ex2(x.x), ex2(x.y));
      ls[c & 1] = add2(ls[c & 1], pp);
      const __half2 hp = __floats2half2_rn(pp.x, pp.y);
      pk[c] = *reinterpret_cast<const uint32_t*>(&hp);
    }
    const float2 lsum = add2(ls[0], ls[1]);
    l += lsum.x + lsum.y;
    if (tt > 0) {
      // P's columns (and O) are free once the CTA's previous PV has completed;
      // the first tile of a unit leaves O alone (its PV overwrites it)
      if (!warp_wait(smem_u32(&B->pv_done), static_cast<uint32_t>(tt - 1) & 1u, B)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (jj > 0 && __any_sync(0xffffffffu, need)) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t v[32];
          tmem_ld32(lane_base + kColO + 64 * wg + 32 * c, v);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float2 o2 = mul2(make_float2(__uint_as_float(v[i]), __uint_as_float(v[i + 1])),
                                   make_float2(factor, factor));
            v[i] = __float_as_uint(o2.x);
            v[i + 1] = __float_as_uint(o2.y);
          }
          tmem_st32(lane_base + kColO + 64 * wg + 32 * c, v);
        }
      }
    }
    tmem_st32(lane_base + kColP + 32 * wg, pk);
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&B->p_full));
  }
  if (ok && !warp_wait(smem_u32(&B->pv_done), static_cast<uint32_t>(T + w.n - 1) & 1u, B)) ok = false;
  // both halves of l through their own slots; every thread arrives on every
  // path (a fast warpgroup writes these slots again only after the next
  // unit's maximum exchanges, which the slow one joins after reading them)
  float* lslot = reinterpret_cast<float*>(smem + kOffL);
  lslot[wg * kRows + r] = l;
  mbar_arrive(smem_u32(&B->l_full));
  if (ok && !warp_wait(smem_u32(&B->l_full), static_cast<uint32_t>(i) & 1u, B)) ok = false;
  l = lslot[r] + lslot[kRows + r];
  if (!ok) return false;
  tc_fence_after();
  // O out of TMEM (complete before this warp's next P store and p_full
  // arrival, which the next unit's first PV, overwriting O, waits for)
  uint32_t v0[32], v1[32];
  tmem_ld32(lane_base + kColO + 64 * wg, v0);
  tmem_ld32(lane_base + kColO + 64 * wg + 32, v1);
  tmem_wait_ld();
  // out = O e^(m - M) / (l e^(m - M) + e^(sink - M)), M = max(m, sink), in log2 units
  const float s2 = p.sinks[h] * kPfLog2e;
  const float M = fmaxf(m, s2);
  const float a = (m == -INFINITY) ? 0.f : ex2(m - M);
  const float sc = a / (l * a + ex2(s2 - M));
  // The scaled O goes out through a per-warp staging tile, 16 of this
  // warpgroup's 64 dims per round: each lane writes its row (16-byte chunks
  // swizzled by row so that a quarter-warp hits distinct banks), then every
  // store instruction covers 64 contiguous bytes of 8 rows (rows 8k..8k+7 are
  // the 8 heads of one token, 512 bytes apart).  Lane-per-row stores would
  // touch 32 lines per instruction.
  float* stg = reinterpret_cast<float*>(smem + kOffStage + warp * kStageWarpBytes);
  const int row0 = (warp & 3) * 32;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
#pragma unroll
    for (int i4 = 0; i4 < 4; ++i4) {
      const int e = (q & 1) * 16 + 4 * i4;
      const float4 val = q < 2 ? make_float4(__uint_as_float(v0[e]) * sc, __uint_as_float(v0[e + 1]) * sc,
                                             __uint_as_float(v0[e + 2]) * sc, __uint_as_float(v0[e + 3]) * sc)
                               : make_float4(__uint_as_float(v1[e]) * sc, __uint_as_float(v1[e + 1]) * sc,
                                             __uint_as_float(v1[e + 2]) * sc, __uint_as_float(v1[e + 3]) * sc);
      reinterpret_cast<float4*>(stg + lane * 16)[i4 ^ ((lane >> 1) & 3)] = val;
    }
    __syncwarp();
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int rw = 8 * k + (lane >> 2), c4 = lane & 3;  // row of the warp, 16-byte chunk
      const float4 val = reinterpret_cast<const float4*>(stg + rw * 16)[c4 ^ ((rw >> 1) & 3)];
      const int rr = row0 + rw;
      const int tr = w.t0 + (rr >> 3);
      if (tr < p.T)
        *reinterpret_cast<float4*>(p.out + (static_cast<long long>(tr) * kHeads + w.g * kGroup + (rr & 7)) * kDim +
                                   64 * wg + 16 * q + 4 * c4) = val;
    }
    __syncwarp();
  }
  return true;
}

// The softmax warps over the CTA's units.
__device__ void run_softmax(const PrefillParams& p, uint32_t tmem, uint8_t* smem, Bars* B, int warp, int lane) {
  const int units = n_units(p);
  int T = 0;
  for (int i = 0;; ++i) {
    const int u = unit_of(i);
    if (u >= units) break;
    const Work w = work_of_unit(p, u);
    if (!softmax_unit(p, w, i, T, tmem, smem, B, warp, lane)) {
      if (lane == 0) raise_abort(p, B);
      return;
    }
    T += w.n;
  }
}

__global__ void __launch_bounds__(kPfThreads, 1) prefill_kernel(const __grid_constant__ PrefillParams p) {
  extern __shared__ uint8_t pf_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(pf_raw) + 1023) & ~uintptr_t(1023));
  Bars* B = reinterpret_cast<Bars*>(smem + kOffBar);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&B->q_full), 1);
    mbar_init(smem_u32(&B->q_empty), 1);
    for (int s = 0; s < kKs; ++s) {
      mbar_init(smem_u32(&B->k_full[s]), 1);
      mbar_init(smem_u32(&B->k_empty[s]), 1);
    }
    for (int s = 0; s < kVs; ++s) {
      mbar_init(smem_u32(&B->v_full[s]), 1);
      mbar_init(smem_u32(&B->v_empty[s]), 1);
    }
    mbar_init(smem_u32(&B->s_full[0]), 1);
    mbar_init(smem_u32(&B->s_full[1]), 1);
    mbar_init(smem_u32(&B->p_full), kSoftWarps);
    mbar_init(smem_u32(&B->pv_done), 1);
    mbar_init(smem_u32(&B->mma_done), 1);
    mbar_init(smem_u32(&B->red_full[0]), kSoftWarps * 32);
    mbar_init(smem_u32(&B->red_full[1]), kSoftWarps * 32);
    mbar_init(smem_u32(&B->l_full), kSoftWarps * 32);
    B->abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == kTmaWarp && lane == 0) {
    prefetch_tensormap(&p.q_map);
    prefetch_tensormap(&p.k_map);
    prefetch_tensormap(&p.v_map);
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(&B->tmem_base))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = B->tmem_base;

  Issued issued{0, 0, 0};
  if (warp < kSoftWarps) {
    run_softmax(p, tmem, smem, B, warp, lane);
  } else if (warp == kTmaWarp) {
    if (lane == 0) issued = run_tma(p, smem, B);
  } else if (lane == 0) {
    run_mma(p, smem_u32(smem), tmem, B);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kTmaWarp && lane == 0 && aborted(B)) drain_tma(issued, B);
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
  }
}

}  // namespace

#ifdef FLINT_TEST_HOOKS
// Test builds only: both exponentials of the softmax, ex2_fma2 (pairs x[2i],
// x[2i+1]; a last odd element paired with itself) and ex2.approx, of n values
// (device pointers), for the comparison in the tests.
__global__ void ex2_probe_kernel(const float* x, float* y_fma, float* y_mufu, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i < n) {
    const float a = x[i], b = i + 1 < n ? x[i + 1] : a;
    const float2 y = ex2_fma2(make_float2(a, b));
    y_fma[i] = y.x;
    y_mufu[i] = ex2(a);
    if (i + 1 < n) {
      y_fma[i + 1] = y.y;
      y_mufu[i + 1] = ex2(b);
    }
  }
}
extern "C" int flint_test_ex2(const float* x, float* y_fma, float* y_mufu, int n, void* stream) {
  if (n < 1) return static_cast<int>(cudaErrorInvalidValue);
  const int pairs = (n + 1) / 2;
  ex2_probe_kernel<<<(pairs + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y_fma, y_mufu, n);
  return static_cast<int>(cudaGetLastError());
}

// Test builds only: CTA `block` leaves its K tile `tile` unarmed; block = -1
// turns the hook off.
extern "C" int flint_test_stall_prefill(int block, int tile) {
  const int v[2] = {block, tile};
  return static_cast<int>(cudaMemcpyToSymbol(g_stall_prefill, v, sizeof v));
}
#endif

cudaError_t launch_prefill(const PrefillParams& p, int num_sms, cudaStream_t stream) {
  static ContextSet configured;
  cudaError_t e = configure_once(configured, reinterpret_cast<const void*>(prefill_kernel), static_cast<int>(kPfSmem));
  if (e != cudaSuccess) return e;
  // one persistent CTA per SM (the kernel fills an SM's TMEM), at most one per unit
  const int grid = std::min((p.T + kPq - 1) / kPq * kKvHeads, num_sms);
  prefill_kernel<<<grid, kPfThreads, kPfSmem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace flint
