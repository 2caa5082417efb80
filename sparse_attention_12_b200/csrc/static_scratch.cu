// dsa_layer_noalloc: the whole path without caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they run a layer: code that runs
// while a memory pool is locked or being defragmented, allocator-free embedded runtimes, and hooks
// that must not call cudaMalloc (which can synchronise the device). This entry point takes the
// same inputs and outputs as dsa_layer but carves its workspace (batch plan, score rows, index
// sets, split partials) out of one file-scope device array instead.
//
// The array is kStaticScratchBytes (64 MiB) per device; every GPU that loads the library holds it
// until the process exits. Its device address is looked up with cudaGetSymbolAddress on every
// call (a host-side query; the address can change if the device's primary context is torn down
// and created again). The first call on a device also loads the library's device code there:
// make that first call before any stream capture.
// All calls share the array and it keeps the last call's contents: calls whose kernels overlap
// on the GPU (different streams, or several host threads) race on it. Nothing in it needs to
// start at zero: the plan kernel rewrites the status word and every other region is written
// before it is read. The plan, with the status word the kernels record run-time faults in, sits at
// the start of the array; dsa_layer_noalloc_status_read reads (and clears) that word.
#include <cuda_runtime.h>

#include "dsa_internal.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(64) << 20;

__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of g_static_scratch on the current device (nullptr on failure).
void* scratch_for_current_device() {
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_static_scratch) != cudaSuccess) return nullptr;
  return ptr;
}

}  // namespace

extern "C" dsa_status_t dsa_layer_noalloc(const dsa_batch_t* batch, const uint8_t* qI, const float* qI_scale,
                                          const float* wI, int nhI, const uint8_t* kI_cache, const float* kI_scale,
                                          const void* q, int H, const void* kv_cache, int k, float softmax_scale,
                                          void* out, float* lse, int32_t* S_out, void* stream) {
  // the same argument checks, in the same order, as dsa_layer; then the size limit
  const dsa_status_t st = dsa::check_layer_args(batch, qI, qI_scale, wI, nhI, kI_cache, kI_scale, q, H, kv_cache,
                                                k, softmax_scale, out);
  if (st != DSA_OK || batch->total_q == 0) return st;
  const size_t need = dsa_layer_workspace_size(batch, nhI, H, k);
  if (need == 0) return DSA_ERR_INVALID_ARG;  // unreachable once the checks above passed
  if (need > kStaticScratchBytes) return DSA_ERR_WORKSPACE;
  void* ws = scratch_for_current_device();
  if (!ws) return DSA_ERR_CUDA;
  return dsa_layer(batch, qI, qI_scale, wI, nhI, kI_cache, kI_scale, q, H, kv_cache, k, softmax_scale, out, lse,
                   S_out, ws, kStaticScratchBytes, stream);
}

extern "C" dsa_status_t dsa_layer_noalloc_status_read(void* stream) {
  void* ws = scratch_for_current_device();
  if (!ws) return DSA_ERR_CUDA;
  return dsa_status_read(ws, stream);
}
