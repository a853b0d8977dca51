// flint_device.cuh -- device helpers: inline PTX for TMA, mbarriers,
// ldmatrix and bf16 mma.sync, bounded waits, and the per-row Q/K norm+RoPE.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "flint_internal.h"

namespace flint {

// A pipeline wait gives up after this long (the whole decode step takes well
// under a millisecond); the kernel then reports FLINT_ERR_TIMEOUT.  A build
// for the time-out tests sets a short limit (FLINT_WAIT_LIMIT_NS).
#ifndef FLINT_WAIT_LIMIT_NS
#define FLINT_WAIT_LIMIT_NS 2000000000ull
#endif
constexpr unsigned long long kWaitLimitNs = FLINT_WAIT_LIMIT_NS;

// Test hooks (FLINT_TEST_HOOKS, only together with FLINT_DEBUG_CHECKS): a
// kernel can be told to leave one pipeline stage of one CTA unarmed, so that
// the waits on it run out and the abort path runs without any fault.
#if defined(FLINT_TEST_HOOKS) && !defined(FLINT_DEBUG_CHECKS)
#error "FLINT_TEST_HOOKS needs FLINT_DEBUG_CHECKS"
#endif

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void report_error(int32_t* dev_err, int code) {
  if (dev_err) atomicCAS(dev_err, 0, code);
}

// ---- self-checks (FLINT_DEBUG_CHECKS builds only) ---------------------------
// A failed check records (code, block, thread, a, b, c) in dev_err[2..7] once
// and the caller skips the access; release builds compile the checks away.
#ifdef FLINT_DEBUG_CHECKS
static __device__ __noinline__ void debug_record(int32_t* rec, int code, int a, int b, int c) {
  if (rec && atomicCAS(rec + 2, 0, code) == 0) {
    rec[3] = blockIdx.x;
    rec[4] = threadIdx.x;
    rec[5] = a;
    rec[6] = b;
    rec[7] = c;
  }
}
#define FLINT_CHECK(rec, cond, code, a, b, c) \
  ((cond) ? true : (::flint::debug_record((rec), (code), (a), (b), (c)), false))
#else
#define FLINT_CHECK(rec, cond, code, a, b, c) ((void)(rec), true)
#endif

// ---- mbarrier -------------------------------------------------------------

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete.  Returns false if the
// CTA's abort flag is raised or the time limit passes.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity,
                                          const volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  }
}

// ---- TMA ------------------------------------------------------------------

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

// The same load with an L2 eviction-priority hint (a policy from
// l2_policy_evict_first): the KV cache is read once per call, so its lines
// should leave the L2 before data that is read again (split partials).
__device__ __forceinline__ void tma_load_4d_hint(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                                 int c0, int c1, int c2, int c3, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4, %5, %6}], [%2], %7;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// Plain bulk copy global -> shared (16-byte aligned, size a multiple of 16),
// completing on an mbarrier.
__device__ __forceinline__ void bulk_copy_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                              uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Order this thread's generic-proxy global writes before later async-proxy
// (TMA) reads of the same addresses.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// ---- ldmatrix / mma.sync ---------------------------------------------------

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                          uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D (16x8 fp32) += A (16x16 bf16, row) * B (16x8 bf16, col).
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D (16x8 fp32) += A (16x16 fp16, row) * B (16x8 fp16, col).
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                              uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Transpose of an 8x8 b16 matrix held one fragment per lane (lane t: row t/4,
// columns 2(t%4), 2(t%4)+1) into the same fragment layout.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// ---- E4M3 helpers -----------------------------------------------------------

// Four E4M3 codes (byte i = code i) -> two packed f16x2: codes 0, 1 in `lo`,
// codes 2, 3 in `hi` (first of each pair in the low half); the two 16-bit
// halves of the word feed the conversions directly.
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t four, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, a;\n\tcvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(four));
}

// Two floats -> two E4M3 codes (first in the low byte), nearest even,
// saturating at +-448.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float a, float b) {
  return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3));
}

// x = hi + lo with hi = f16(x), lo = f16(x - hi), as split_bf16x2 for f16
// operands (~22 significant bits for magnitudes well inside the f16 range).
__device__ __forceinline__ void split_f16x2(float a, float b, uint32_t& hi, uint32_t& lo) {
  const __half2 h = __floats2half2_rn(a, b);
  const float2 hf = __half22float2(h);
  const __half2 l = __floats2half2_rn(a - hf.x, b - hf.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

// ---- paired fp32 arithmetic (sm_100) -----------------------------------------

// Paired fp32 arithmetic (one instruction for two lanes of a float2, each
// rounded to nearest as the scalar operation would be).
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mov.b64 rc, {%6, %7};\n\tfma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
// max(a, b, c) in one instruction (as fmaxf(fmaxf(a, b), c)).
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// ---- bf16 helpers ----------------------------------------------------------

__device__ __forceinline__ float bf16_lo(uint32_t packed) {
  return __uint_as_float(packed << 16);
}
__device__ __forceinline__ float bf16_hi(uint32_t packed) {
  return __uint_as_float(packed & 0xffff0000u);
}

// Two floats -> packed bf16x2 (first in the low half), round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

// x = hi + lo with hi = bf16(x), lo = bf16(x - hi): a two-term bf16 split that
// carries ~16 significant bits into a bf16 tensor-core product.
__device__ __forceinline__ void split_bf16x2(float a, float b, uint32_t& hi, uint32_t& lo) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  float2 hf = __bfloat1622float2(h);
  __nv_bfloat162 l = __floats2bfloat162_rn(a - hf.x, b - hf.y);
  hi = *reinterpret_cast<uint32_t*>(&h);
  lo = *reinterpret_cast<uint32_t*>(&l);
}

// ---- per-head RMSNorm (+RoPE) of one 128-wide row by one warp ---------------
// Lane l holds dims (2l, 2l+1, 64+2l, 65+2l): RoPE pairs (i, i+64) stay in one
// lane.  y = x * w / sqrt(mean(x^2) + eps), then for i < 64 the pair
// (y_i, y_{i+64}) turns by the angle whose cos/sin are cs[i].
__device__ __forceinline__ void norm_rope_row_warp(const uint16_t* __restrict__ x_row,
                                                   const uint16_t* __restrict__ w, float eps,
                                                   bool do_norm, bool rope, const float2* cs,
                                                   int lane, float (&y)[4]) {
  const uint32_t xa = reinterpret_cast<const uint32_t*>(x_row)[lane];
  const uint32_t xb = reinterpret_cast<const uint32_t*>(x_row + 64)[lane];
  y[0] = bf16_lo(xa);
  y[1] = bf16_hi(xa);
  y[2] = bf16_lo(xb);
  y[3] = bf16_hi(xb);
  if (do_norm) {
    float ss = y[0] * y[0] + y[1] * y[1] + y[2] * y[2] + y[3] * y[3];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float r = 1.0f / sqrtf(ss * (1.0f / kDim) + eps);
    const uint32_t wa = reinterpret_cast<const uint32_t*>(w)[lane];
    const uint32_t wb = reinterpret_cast<const uint32_t*>(w + 64)[lane];
    y[0] = y[0] * r * bf16_lo(wa);
    y[1] = y[1] * r * bf16_hi(wa);
    y[2] = y[2] * r * bf16_lo(wb);
    y[3] = y[3] * r * bf16_hi(wb);
  }
  if (rope) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float2 t = cs[2 * lane + e];
      const float a = y[e], b = y[2 + e];
      y[e] = a * t.x - b * t.y;
      y[2 + e] = b * t.x + a * t.y;
    }
  }
}

// cos/sin of pos * theta^(-2i/128) for i < 64, angle formed and reduced in
// double precision (an fp32 angle near position 1e5 would be off by ~1e-2 rad).
__device__ __forceinline__ float2 rope_cos_sin(int i, int pos, double theta) {
  const double inv_freq = pow(theta, -2.0 * i / kDim);
  double s, c;
  sincos(static_cast<double>(pos) * inv_freq, &s, &c);
  return make_float2(static_cast<float>(c), static_cast<float>(s));
}

}  // namespace flint
