// Decode entry point for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc where they run a decode step: an
// inference engine that reserves its device memory once at start-up and
// forbids allocation inside the step loop, a plugin that runs under another
// framework's memory manager, or a latency-critical loop where an allocation
// call could synchronise the device.  mxa_decode_fwd_noalloc serves them: it
// runs the same split kernel and merge as mxa_decode_fwd, but its split
// results live in one fixed array inside this library instead of a
// caller-provided workspace.
#include <cuda_runtime.h>

#include <mutex>

#include "mxa.h"

namespace {

// Upper bound on the scratch a plan may need here (16 MiB).  The array is
// part of the library's device image: every GPU that loads the library holds
// it until the process exits.
constexpr size_t kNoAllocScratchBytes = (size_t)16 << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of the array on the current device.  The name of a
// __device__ array in host code is only a host-side stand-in, so the address
// is looked up once per device (with that device current) and cached.
mxa_status_t scratch_address(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MXA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return MXA_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return MXA_OK;
}

}  // namespace

extern "C" mxa_status_t mxa_decode_fwd_noalloc(const void *q, const void *k_cache, const void *v_cache,
                                               const int32_t *block_table, const int32_t *cache_seqlens,
                                               const mxa_decode_params_t *params, float scale, int causal,
                                               int num_splits, void *out, float *lse, void *stream) {
  mxa_plan_t plan;
  mxa_status_t st = mxa_plan(params, num_splits, 0, &plan);
  if (st != MXA_OK) return st;
  if (plan.workspace_bytes > kNoAllocScratchBytes) return MXA_ERR_WORKSPACE;  // past the fixed array
  void *scratch = nullptr;
  if (plan.workspace_bytes > 0) {
    st = scratch_address(&scratch);
    if (st != MXA_OK) return st;
  }
  return mxa_decode_fwd_with_plan(q, k_cache, v_cache, block_table, cache_seqlens, params, scale, causal,
                                  &plan, scratch, kNoAllocScratchBytes, out, lse, stream);
}
