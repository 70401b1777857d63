// pa_noalloc.cu -- pa_decode_noalloc: pa_decode for callers that cannot
// allocate device memory.
//
// pa_decode keeps its split-K partials (per-partition maxima, sums and partial
// outputs) in a workspace the caller allocates.  Some callers cannot do that:
// code running inside another framework's allocator, plugins that are handed
// only input and output buffers, or hosts that must not call cudaMalloc on
// their hot path.  For them this entry point keeps the partials in a fixed
// array compiled into the library (PA_NOALLOC_SCRATCH_BYTES, 32 MiB per GPU,
// held by every GPU that loads the library until the process exits).
//
// Rules of use:
//  - The first call on each device looks up the array's device address
//    (cudaGetSymbolAddress, with that device current); make that first call
//    before any stream capture.  After cudaDeviceReset the first call in the
//    new context looks it up again (the reset reloads the module).
//  - Every call on a device shares the one array, so calls whose kernels
//    overlap on the GPU (different streams, no ordering between them) race.
//  - Nothing in the array has to start at zero: each call reads only the
//    partials it wrote earlier in the same call.
//  - A call that needs more scratch than the array holds is rejected with
//    PA_ERR_WORKSPACE before anything is launched.
//  - Nothing here calls cudaMalloc, cudaFree or any allocating routine.
#include <cstdio>
#include <mutex>

#include <cuda_runtime.h>

#include "../../include/pagedattn.h"
#include "pa_kernels.cuh"

// The scratch array (file scope, internal linkage).
static __device__ __align__(256) unsigned char g_noalloc_scratch[PA_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 128;

// Device address of g_noalloc_scratch on the current device.  In host code
// the array's name is only a host-side stand-in, so the kernels are given
// this address instead.  It is looked up with the device current, once per
// device and CUDA context: cudaDeviceReset replaces the device's context and
// reloads the library's module, which moves the array, so a call made in a
// new context looks the address up again.
int scratch_address(void** out) {
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  static unsigned long long ctx_of[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    fprintf(stderr, "pa_decode_noalloc: cannot read the current device\n");
    return PA_ERR_CUDA;
  }
  const unsigned long long ctx = pa::context_id();
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev] || ctx == 0 || ctx != ctx_of[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) {
      fprintf(stderr, "pa_decode_noalloc: cudaGetSymbolAddress failed: %s\n",
              cudaGetErrorString(e));
      return PA_ERR_CUDA;
    }
    addr[dev] = p;
    ctx_of[dev] = pa::context_id();  // the lookup itself may have created the context
  }
  *out = addr[dev];
  return PA_OK;
}

}  // namespace

extern "C" {

// pa_decode with the static array as its workspace.  pa_decode's own check
// rejects, before launching anything, a call whose partials need more than
// PA_NOALLOC_SCRATCH_BYTES (PA_ERR_WORKSPACE, message in pa_last_error()).
int pa_decode_noalloc(void* dst, const void* q, const void* kCache, const void* vCache,
                      const int32_t* blockTables, const int32_t* seqLens,
                      const int32_t* queryLens, float scale, int window, int kvBlockSize,
                      const pa_params* params, void* stream) {
  if (!params)
    return pa_decode(dst, q, kCache, vCache, blockTables, seqLens, queryLens, scale, window,
                     kvBlockSize, params, stream);
  pa_params p = *params;
  int rc = scratch_address(&p.workspace);
  if (rc) return rc;
  p.workspace_bytes = PA_NOALLOC_SCRATCH_BYTES;
  return pa_decode(dst, q, kCache, vCache, blockTables, seqLens, queryLens, scale, window,
                   kvBlockSize, &p, stream);
}

}  // extern "C"
