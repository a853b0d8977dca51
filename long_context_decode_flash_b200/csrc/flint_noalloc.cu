// flint_noalloc.cu -- flint_attn_stack_noalloc: the 49-layer stack call for
// callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at all at the moment they decode: a
// runtime that owns every byte of the GPU through its own pool, a plug-in that
// is handed buffers but no allocator, or code that must not allocate once it
// has started.  flint_attn_stack asks them for a workspace; this entry point
// instead uses a scratch array that the library itself holds in device memory
// for as long as it is loaded.
//
// The scratch is one file-scope device array of FLINT_NOALLOC_SCRATCH_BYTES.
// Every device on which the library's device code is loaded holds a copy
// until the process exits.  All calls on a device share that one copy, and
// it keeps whatever the last call left in it.  Two calls whose launches
// overlap on the GPU (two streams, or two host threads) race on it and give
// wrong results; order them on one stream or use flint_attn_stack with a
// workspace each.
//
// Set-up: the first call on a device, made with that device current, looks up
// the address of the device's copy of the scratch (cudaGetSymbolAddress) and
// keeps it for later calls.  Make that first call before any stream capture.
// The address belongs to the device's current CUDA context: after a device
// reset the runtime makes a new context, the next call looks the address up
// again, and that call too must come before any capture.
#include <cuda_runtime.h>
#include <stdio.h>

#include <mutex>

#include "flint_internal.h"

using namespace flint;

namespace {

static_assert(FLINT_NOALLOC_SCRATCH_BYTES % 256 == 0, "scratch size is a multiple of 256 bytes");
static_assert(FLINT_NOALLOC_SCRATCH_BYTES > kCounterBytes, "scratch holds the counters and partials");

// The scratch: the counter area (arrival counters, grid-barrier, queue,
// abort and merge-ticket words, item ready flags) in its first
// kCounterBytes, split partials after them (the workspace layout of
// flint_attn_stack).
static __device__ __align__(256) unsigned char g_scratch[FLINT_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};
void* g_scratch_ctx[kMaxDevices] = {};  // the context each address was looked up in

// Address of the current device's copy of g_scratch.  The first call on a
// device looks it up (with that device current) and keeps it together with the
// current context; a call in another context (after a device reset) looks it
// up again.
flint_status scratch_address(void** out, const char* who) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return record_error(FLINT_ERR_CUDA, "%s: cudaGetDevice failed: %s", who, cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices)
    return record_error(FLINT_ERR_UNSUPPORTED, "%s: device %d outside the %d devices supported", who, dev, kMaxDevices);
  std::lock_guard<std::mutex> lock(g_mu);
  void* ctx = current_context();
  if (!g_scratch_addr[dev] || !ctx || ctx != g_scratch_ctx[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess || !p)
      return record_error(FLINT_ERR_CUDA, "%s: cudaGetSymbolAddress of the scratch failed on device %d: %s",
                          who, dev, cudaGetErrorString(e));
    g_scratch_addr[dev] = p;
    g_scratch_ctx[dev] = current_context();  // the lookup above made one if there was none
  }
  *out = g_scratch_addr[dev];
  return FLINT_OK;
}

}  // namespace

extern "C" flint_status flint_attn_stack_noalloc(const flint_layer* layers, int32_t n_layers,
                                                 int32_t pos, float eps, double theta, float* out,
                                                 int32_t num_ctas, int32_t* dev_err, void* stream) {
  const char* who = "flint_attn_stack_noalloc";
  FLINT_NVTX_RANGE(who);
  // Size check first: the scratch cannot grow.  It must hold the static plan;
  // the run-time queue then gets the part of it that is left.
  const size_t need = workspace_min_bytes(n_layers, num_ctas);
  if (need == 0)
    return record_error(FLINT_ERR_INVALID_ARG, "%s: n_layers=%d or num_ctas=%d out of range", who, n_layers, num_ctas);
  if (need > FLINT_NOALLOC_SCRATCH_BYTES)
    return record_error(FLINT_ERR_WORKSPACE,
                        "%s: %d layers with num_ctas=%d (0: one CTA per SM) need %zu bytes of scratch, "
                        "above the fixed %zu; pass fewer CTAs or call flint_attn_stack with a workspace",
                        who, n_layers, num_ctas, need, (size_t)FLINT_NOALLOC_SCRATCH_BYTES);
  void* scratch = nullptr;
  flint_status s = scratch_address(&scratch, who);
  if (s != FLINT_OK) return s;
  // The counters must start at zero; a previous call that ended in a device
  // error can have left them otherwise.  The partials need no clearing: every
  // partial is written before it is read.
  const cudaError_t e = cudaMemsetAsync(scratch, 0, kCounterBytes, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess)
    return record_error(FLINT_ERR_CUDA, "%s: clearing the scratch counters failed: %s", who, cudaGetErrorString(e));
  return flint_attn_stack(layers, n_layers, pos, eps, theta, out, scratch, FLINT_NOALLOC_SCRATCH_BYTES,
                          num_ctas, dev_err, stream);
}
