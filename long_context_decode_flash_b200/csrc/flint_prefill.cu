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
// How: one CTA per (block of 16 query tokens, KV head g); warp w of the CTA
// serves query head 8g + w, so the 8 heads of a GQA group share every K/V
// tile.  64-token K and V tiles of the KV head stream through two shared-
// memory stages with cp.async (16-byte chunks, XOR-swizzled so that ldmatrix
// reads are conflict-free); blocks run from the last (longest) to the first.
// Per tile and warp: S = Q K^T on bf16 mma.sync m16n8k16 (rows = the 16 query
// tokens), the causal / window mask on boundary tiles, an fp32 online softmax
// per row in log2 units, and O += P V with P split into bf16 hi and lo parts
// (two products), so that P keeps ~16 bits.
#include <math.h>

#include "flint_device.cuh"

namespace flint {

namespace {

constexpr int kPfQ = 16;                        // query tokens per CTA
constexpr int kPfKv = 64;                       // key tokens per tile
constexpr int kPfThreads = kGroup * 32;         // one warp per query head of the group
constexpr int kPfRow = kDim * 2;                // bytes of one token's 128 dims of one KV head
constexpr int kPfTile = kPfKv * kPfRow;         // 16 KiB
constexpr int kPfStages = 2;
constexpr size_t kPfSmem = static_cast<size_t>(kPfStages) * 2 * kPfTile;  // K and V: 64 KiB
constexpr float kPfLog2e = 1.4426950408889634f;
constexpr float kPfScale = static_cast<float>(1.4426950408889634 * 0.08838834764831845);

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  // a chunk past the prompt is zero-filled (source size 0; the address stays in bounds)
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Loads tile j of KV head g (keys 64j .. 64j + 63) into stage buffers sK, sV:
// row r, 16-byte chunk u goes to r * 256 + ((u ^ (r & 7)) << 4).
__device__ __forceinline__ void load_tile(const PrefillParams& p, int g, int j, uint32_t sK, uint32_t sV) {
  for (int ch = threadIdx.x; ch < kPfKv * (kPfRow / 16); ch += kPfThreads) {
    const int r = ch >> 4, u = ch & 15;
    const int key = j * kPfKv + r;
    const bool valid = key < p.T;
    const long long off = (static_cast<long long>(valid ? key : 0) * kKvHeads + g) * kDim + u * 8;
    const uint32_t so = static_cast<uint32_t>(r * kPfRow + ((u ^ (r & 7)) << 4));
    cp_async16(sK + so, p.k + off, valid);
    cp_async16(sV + so, p.v + off, valid);
  }
}

__global__ void __launch_bounds__(kPfThreads, 1) prefill_kernel(const __grid_constant__ PrefillParams p) {
  extern __shared__ __align__(1024) uint8_t pf_smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, c = lane & 3, l7 = lane & 7;
  const int qb = gridDim.x - 1 - blockIdx.x;  // longest blocks first
  const int g = blockIdx.y;
  const int h = g * kGroup + warp;
  const int t0 = qb * kPfQ;
  const int ta = t0 + gq, tb = t0 + gq + 8;    // this thread's two query rows

  // Q fragments (A operand rows: tokens ta and tb), straight from global memory
  uint32_t qa[8][4];
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const int d0 = 16 * kk + 2 * c;
    const uint16_t* qa_row = p.q + (static_cast<long long>(ta < p.T ? ta : 0) * kHeads + h) * kDim;
    const uint16_t* qb_row = p.q + (static_cast<long long>(tb < p.T ? tb : 0) * kHeads + h) * kDim;
    qa[kk][0] = ta < p.T ? *reinterpret_cast<const uint32_t*>(qa_row + d0) : 0u;
    qa[kk][1] = tb < p.T ? *reinterpret_cast<const uint32_t*>(qb_row + d0) : 0u;
    qa[kk][2] = ta < p.T ? *reinterpret_cast<const uint32_t*>(qa_row + d0 + 8) : 0u;
    qa[kk][3] = tb < p.T ? *reinterpret_cast<const uint32_t*>(qb_row + d0 + 8) : 0u;
  }

  const int t_last = min(t0 + kPfQ - 1, p.T - 1);
  const int j_first = p.window > 0 ? max(0, t0 - (p.window - 1)) / kPfKv : 0;
  const int j_last = t_last / kPfKv;
  const uint32_t base = smem_u32(pf_smem);

  float o[16][4];
#pragma unroll
  for (int n = 0; n < 16; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[n][e] = 0.f;
  float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;

  load_tile(p, g, j_first, base, base + kPfTile);
  cp_async_commit();
  for (int j = j_first; j <= j_last; ++j) {
    const int st = (j - j_first) & 1;
    if (j < j_last) {
      const uint32_t nb = base + static_cast<uint32_t>(((j + 1 - j_first) & 1) * 2 * kPfTile);
      load_tile(p, g, j + 1, nb, nb + kPfTile);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const uint32_t sK = base + static_cast<uint32_t>(st * 2 * kPfTile), sV = sK + kPfTile;

    // S = Q K^T for the tile's 64 keys: 8 n-tiles of 8 keys
    float s[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) s[nt][e] = 0.f;
      const uint32_t row = sK + (8 * nt + l7) * kPfRow;
#pragma unroll
      for (int kk = 0; kk < 8; kk += 2) {
        const int u = 2 * kk + (lane >> 3);  // 16-byte chunk: dims 8u .. 8u + 7
        uint32_t b0, b1, b2, b3;
        ldsm_x4(row + ((u ^ l7) << 4), b0, b1, b2, b3);
        mma_bf16_16816(s[nt], qa[kk], b0, b1);
        mma_bf16_16816(s[nt], qa[kk + 1], b2, b3);
      }
    }
    // scale to log2 units; mask keys past a row's position, before its window or past the prompt
    const int k0 = j * kPfKv;
    const bool interior = (k0 + kPfKv - 1 <= t0) && (k0 + kPfKv <= p.T) &&
                          (p.window == 0 || k0 > t_last - p.window);
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        s[nt][e] *= kPfScale;
        if (!interior) {
          const int key = k0 + 8 * nt + 2 * c + (e & 1);
          const int t = (e < 2) ? ta : tb;
          const bool ok = key <= t && key < p.T && (p.window == 0 || key > t - p.window);
          if (!ok) s[nt][e] = -INFINITY;
        }
      }
    // online softmax, rows ta (e = 0, 1) and tb (e = 2, 3)
    float mx_a = -INFINITY, mx_b = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      mx_a = fmaxf(mx_a, fmaxf(s[nt][0], s[nt][1]));
      mx_b = fmaxf(mx_b, fmaxf(s[nt][2], s[nt][3]));
    }
    mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 1));
    mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 2));
    mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 1));
    mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 2));
    const float mn_a = fmaxf(m_a, mx_a), mn_b = fmaxf(m_b, mx_b);
    const float al_a = (m_a == -INFINITY) ? 0.f : exp2f(m_a - mn_a);
    const float al_b = (m_b == -INFINITY) ? 0.f : exp2f(m_b - mn_b);
    m_a = mn_a;
    m_b = mn_b;
    l_a *= al_a;
    l_b *= al_b;
#pragma unroll
    for (int n = 0; n < 16; ++n) {
      o[n][0] *= al_a;
      o[n][1] *= al_a;
      o[n][2] *= al_b;
      o[n][3] *= al_b;
    }
    const float mu_a = (m_a == -INFINITY) ? 0.f : m_a, mu_b = (m_b == -INFINITY) ? 0.f : m_b;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      s[nt][0] = exp2f(s[nt][0] - mu_a);
      s[nt][1] = exp2f(s[nt][1] - mu_a);
      s[nt][2] = exp2f(s[nt][2] - mu_b);
      s[nt][3] = exp2f(s[nt][3] - mu_b);
      l_a += s[nt][0] + s[nt][1];
      l_b += s[nt][2] + s[nt][3];
    }

    // O += P V: 4 k-steps of 16 keys, 16 n-tiles of 8 dims, P as bf16 hi + lo
#pragma unroll
    for (int kt = 0; kt < 4; ++kt) {
      uint32_t ph[4], pl[4];
      split_bf16x2(s[2 * kt][0], s[2 * kt][1], ph[0], pl[0]);
      split_bf16x2(s[2 * kt][2], s[2 * kt][3], ph[1], pl[1]);
      split_bf16x2(s[2 * kt + 1][0], s[2 * kt + 1][1], ph[2], pl[2]);
      split_bf16x2(s[2 * kt + 1][2], s[2 * kt + 1][3], ph[3], pl[3]);
      const uint32_t rowv = sV + (16 * kt + ((lane >> 3) & 1) * 8 + l7) * kPfRow;
#pragma unroll
      for (int np = 0; np < 8; ++np) {
        const int u = 2 * np + (lane >> 4);
        uint32_t v0, v1, v2, v3;
        ldsm_x4_t(rowv + ((u ^ l7) << 4), v0, v1, v2, v3);
        mma_bf16_16816(o[2 * np], ph, v0, v1);
        mma_bf16_16816(o[2 * np], pl, v0, v1);
        mma_bf16_16816(o[2 * np + 1], ph, v2, v3);
        mma_bf16_16816(o[2 * np + 1], pl, v2, v3);
      }
    }
    __syncthreads();  // the stage is refilled two tiles later
  }

  // finish: quad-reduce l, fold in the sink, write both rows
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
  const float s2 = p.sinks[h] * kPfLog2e;
  const float Ma = fmaxf(m_a, s2), Mb = fmaxf(m_b, s2);
  const float aa = (m_a == -INFINITY) ? 0.f : exp2f(m_a - Ma), ab = (m_b == -INFINITY) ? 0.f : exp2f(m_b - Mb);
  const float sca = aa / (l_a * aa + exp2f(s2 - Ma)), scb = ab / (l_b * ab + exp2f(s2 - Mb));
  if (ta < p.T) {
    float* out = p.out + (static_cast<long long>(ta) * kHeads + h) * kDim + 2 * c;
#pragma unroll
    for (int n = 0; n < 16; ++n) *reinterpret_cast<float2*>(out + 8 * n) = make_float2(o[n][0] * sca, o[n][1] * sca);
  }
  if (tb < p.T) {
    float* out = p.out + (static_cast<long long>(tb) * kHeads + h) * kDim + 2 * c;
#pragma unroll
    for (int n = 0; n < 16; ++n) *reinterpret_cast<float2*>(out + 8 * n) = make_float2(o[n][2] * scb, o[n][3] * scb);
  }
}

}  // namespace

cudaError_t launch_prefill(const PrefillParams& p, cudaStream_t stream) {
  static int configured_device = -1;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (configured_device != dev) {
    e = cudaFuncSetAttribute(prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kPfSmem));
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  const dim3 grid((p.T + kPfQ - 1) / kPfQ, kKvHeads);
  prefill_kernel<<<grid, kPfThreads, kPfSmem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace flint
