// flint_cp.cu -- the merge step of context-parallel decode: n ranks each ran
// the split-KV attention of the same query over their own token range of a
// full layer's cache (flint_attn_decode_partial) and exchanged the partials;
// this folds them, with the head's sink logit, into the attention output.
// For head h, with partial r = (O_r, m_r, l_r) in log2 units and
// s = sink_h log2(e):
//     M = max(s, max_r m_r),
//     out = sum_r 2^(m_r - M) O_r / (2^(s - M) + sum_r 2^(m_r - M) l_r),
// the log-sum-exp merge of split-KV decoding with the sink as one more
// logit that carries no value ("Day-0 Support for Flint on vLLM",
// hnkhoi.com, "Model architecture": learned attention sinks).  With no key
// anywhere and s = -inf (M = -inf) the output is 0.
#include "flint_device.cuh"

namespace flint {

namespace {

constexpr float kCpLog2e = 1.4426950408889634f;

// One CTA per (request, head), one thread per dim; partials [n][B][4160].
__global__ void __launch_bounds__(kDim) merge_kernel(const float* __restrict__ parts, int n, int B,
                                                     const float* __restrict__ sinks, float* __restrict__ out) {
  const int b = blockIdx.x / kHeads, h = blockIdx.x % kHeads, d = threadIdx.x;
  const float s2 = sinks[h] * kCpLog2e;
  float M = s2;
  for (int r = 0; r < n; ++r)
    M = fmaxf(M, parts[(static_cast<size_t>(r) * B + b) * kCpPartialFloats + kHeads * kDim + h]);
  // No key in any partial and a sink of -inf: the softmax has no mass at all;
  // the output is 0 (nothing carries a value), not 0/0.
  if (M == -INFINITY) {
    out[(static_cast<size_t>(b) * kHeads + h) * kDim + d] = 0.f;
    return;
  }
  float L = exp2f(s2 - M), o = 0.f;
  for (int r = 0; r < n; ++r) {
    const float* pr = parts + (static_cast<size_t>(r) * B + b) * kCpPartialFloats;
    const float m = pr[kHeads * kDim + h];
    const float w = (m == -INFINITY) ? 0.f : exp2f(m - M);
    L += w * pr[kHeads * kDim + kHeads + h];
    o += w * pr[h * kDim + d];
  }
  out[(static_cast<size_t>(b) * kHeads + h) * kDim + d] = o / L;
}

}  // namespace

cudaError_t launch_merge_partials(const float* partials, int n_parts, int B, const float* sinks, float* out,
                                  cudaStream_t stream) {
  merge_kernel<<<B * kHeads, kDim, 0, stream>>>(partials, n_parts, B, sinks, out);
  return cudaGetLastError();
}

}  // namespace flint
