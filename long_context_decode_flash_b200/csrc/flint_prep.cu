// flint_prep.cu -- per-head Q/K RMSNorm + RoPE + KV append for a batch of
// requests ("Day-0 Support for Flint on vLLM", newruntime.com, "What
// happened": fused normalization, rotary-position and cache operations;
// hnkhoi.com "Model architecture": per-head Q/K RMSNorm, RoPE on the
// sliding-window layers, NoPE on the full layers).
//
// One CTA per request, eight warps; each warp owns whole 128-wide rows (32 q
// rows, then 4 k rows) with RoPE pairs (i, i+64) in one lane.  k is rounded
// to bf16 (nearest even) once and the same bits go to k_out and the cache; v
// is copied bit for bit.  With do_norm = 0 and no RoPE the kernel is a plain
// bit-exact append of final k and v.  An E4M3 cache receives, for k and v,
// the codes of float32 (value / scale) (nearest even, saturating), where k is
// the float32 normed (roped) value.  (A prompt's tokens, in prefill, go
// through prefill_prep_kernel instead.)
#include "flint_device.cuh"

namespace flint {

namespace {

constexpr int kPrepThreads = 256;

__global__ void __launch_bounds__(kPrepThreads) prep_kernel(const __grid_constant__ PrepParams p) {
  __shared__ float2 cs[64];
  const int b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pos = p.pos[b];
  const int req = b;
  if (p.apply_rope && threadIdx.x < 64) cs[threadIdx.x] = rope_cos_sin(threadIdx.x, pos, p.theta);
  __syncthreads();

  // element offset of this request's new-token row (KV head 0), or -1
  long long row = -1;
  if (p.k_rows) {
    if (p.layout == FLINT_KV_PAGED) {
      const int blk = p.table[static_cast<long long>(req) * p.max_blocks + pos / kBlock];
      if (blk >= 0 && blk < p.num_blocks) {
        row = (static_cast<long long>(blk) * kBlock + pos % kBlock) * kKvHeads * kDim;
      } else if (threadIdx.x == 0) {
        report_error(p.dev_err, FLINT_ERR_INVALID_ARG);
      }
    } else {
      const int slot = p.layout == FLINT_KV_RING ? pos % p.capacity : pos;
      row = static_cast<long long>(req) * p.req_stride + static_cast<long long>(slot) * kKvHeads * kDim;
    }
  }

  const int first = p.q_raw ? 0 : kHeads;
  for (int r = first + warp; r < kHeads + kKvHeads; r += kPrepThreads / 32) {
    const bool is_q = r < kHeads;
    const int hk = r - kHeads;
    const uint16_t* x = is_q ? p.q_raw + (static_cast<long long>(b) * kHeads + r) * kDim
                             : p.k_raw + (static_cast<long long>(b) * kKvHeads + hk) * kDim;
    float y[4];
    norm_rope_row_warp(x, is_q ? p.w_q : p.w_k, p.eps, p.do_norm != 0, p.apply_rope != 0, cs, lane, y);
    if (is_q) {
      if (p.q_out) {
        float* o = p.q_out + (static_cast<long long>(b) * kHeads + r) * kDim;
        reinterpret_cast<float2*>(o)[lane] = make_float2(y[0], y[1]);
        reinterpret_cast<float2*>(o + 64)[lane] = make_float2(y[2], y[3]);
      }
    } else {
      const uint32_t ka = pack_bf16x2(y[0], y[1]), kb = pack_bf16x2(y[2], y[3]);
      if (p.k_out) {
        uint32_t* o = reinterpret_cast<uint32_t*>(p.k_out + (static_cast<long long>(b) * kKvHeads + hk) * kDim);
        o[lane] = ka;
        o[32 + lane] = kb;
      }
      if (row >= 0 && !p.fp8) {
        uint32_t* o = reinterpret_cast<uint32_t*>(p.k_rows + row + hk * kDim);
        o[lane] = ka;
        o[32 + lane] = kb;
      } else if (row >= 0) {
        const float s = p.k_scale[hk];
        uint16_t* o = reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(p.k_rows) + row + hk * kDim);
        o[lane] = static_cast<uint16_t>(f32x2_to_e4m3x2(__fdiv_rn(y[0], s), __fdiv_rn(y[1], s)));
        o[32 + lane] = static_cast<uint16_t>(f32x2_to_e4m3x2(__fdiv_rn(y[2], s), __fdiv_rn(y[3], s)));
      }
    }
  }
  if (row >= 0 && warp < kKvHeads) {
    const uint2* src = reinterpret_cast<const uint2*>(p.v_raw + (static_cast<long long>(b) * kKvHeads + warp) * kDim);
    if (!p.fp8) {
      uint2* dst = reinterpret_cast<uint2*>(p.v_rows + row + warp * kDim);
      dst[lane] = src[lane];
    } else {
      // lane: dims 4l .. 4l+3
      const uint2 x = src[lane];
      const float s = p.v_scale[warp];
      const uint32_t lo = f32x2_to_e4m3x2(__fdiv_rn(bf16_lo(x.x), s), __fdiv_rn(bf16_hi(x.x), s));
      const uint32_t hi = f32x2_to_e4m3x2(__fdiv_rn(bf16_lo(x.y), s), __fdiv_rn(bf16_hi(x.y), s));
      uint32_t* dst = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(p.v_rows) + row + warp * kDim);
      dst[lane] = (lo & 0xffffu) | (hi << 16);
    }
  }
}

}  // namespace

cudaError_t launch_prep(const PrepParams& p, int B, cudaStream_t stream) {
  prep_kernel<<<B, kPrepThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace flint
