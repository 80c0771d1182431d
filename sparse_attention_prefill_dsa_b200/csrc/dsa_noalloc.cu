// dsa_noalloc.cu -- dsa_prefill_layer_noalloc: the whole layer without a
// caller-supplied workspace.
//
// The layer needs scratch memory between its kernels: the float32 score rows
// written by the indexer and read by the top-k, the selected indices, and a
// status word. dsa_prefill_layer takes that scratch from the caller. Some
// callers cannot allocate device memory for it -- for example code that runs
// inside another engine's plugin or callback and is handed only its input and
// output buffers, or code that must not touch the device allocator while a
// memory pool is shared or being captured. For them this file keeps the
// scratch in a fixed-size static device array and runs the same layer path
// on it.
//
// Rules of the static scratch:
//  * it holds kNoallocScratchBytes (32 MiB) on every GPU that loads the
//    library, until the process exits;
//  * its device address is looked up on the first call made with a device
//    current, and again on the first call after that device's context was
//    destroyed and created anew (cudaDeviceReset, or the primary context
//    released and retained again), since the module and the array may then
//    sit elsewhere; those calls should come before any stream capture;
//  * every call on a device uses the same array, so calls that overlap on the
//    GPU (different streams, or different host threads without ordering) race
//    on it; the layer clears its status word and scalars itself at the start
//    of each call, and every score it reads was written earlier in the same
//    call.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include <mutex>

#include "dsa.h"
#include "dsa_internal.cuh"

namespace {

constexpr size_t kNoallocScratchBytes = static_cast<size_t>(DSA_NOALLOC_SCRATCH_BYTES);
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices];
unsigned long long g_scratch_ctx[kMaxDevices];  // id of the context the address belongs to

PFN_cuCtxGetCurrent_v4000 g_ctx_current = nullptr;
PFN_cuCtxGetId_v12000 g_ctx_id = nullptr;
std::once_flag g_once;

void resolve_driver() {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
  if (cudaGetDriverEntryPoint("cuCtxGetId", &fn, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_ctx_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(fn);
}

// Unique id of the current context (0 when it cannot be read).
unsigned long long current_context_id() {
  std::call_once(g_once, resolve_driver);
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!g_ctx_current || !g_ctx_id || g_ctx_current(&ctx) != CUDA_SUCCESS || !ctx ||
      g_ctx_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of g_noalloc_scratch on the current device (host code only
// sees a host-side stand-in for the symbol, never its device address).
dsa_status scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DSA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return DSA_ERR_DEVICE;
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev] || ctx == 0 || g_scratch_ctx[dev] != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      cudaGetLastError();  // reset the runtime's last-error state after the failed lookup
      return DSA_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = ctx;
  }
  *out = g_scratch_ptr[dev];
  return DSA_OK;
}

}  // namespace

extern "C" dsa_status dsa_prefill_layer_noalloc(const dsa_dims* dims, const uint16_t* q,
                                                const uint16_t* latent, const uint16_t* rope,
                                                const uint16_t* q_idx, const uint16_t* k_idx,
                                                const float* w_idx, uint16_t* out, float* lse,
                                                int32_t* idx_out, uint32_t* device_status,
                                                void* stream) {
  // Argument checks of the layer itself: with no workspace, dsa_prefill_layer
  // returns DSA_ERR_WORKSPACE exactly when every other argument is valid, and
  // it launches nothing in either case.
  dsa_status s = dsa_prefill_layer(dims, q, latent, rope, q_idx, k_idx, w_idx, out, lse, idx_out,
                                   nullptr, 0, stream);
  if (s != DSA_ERR_WORKSPACE) return s;
  if (dsa_workspace_size(dims, DSA_WS_LAYER) > kNoallocScratchBytes) return DSA_ERR_SCRATCH_LIMIT;
  if (device_status && (reinterpret_cast<uintptr_t>(device_status) & 3u) != 0)
    return DSA_ERR_ALIGN;
  // a GPU this library was not built for fails here, before the symbol lookup
  if ((s = dsa::check_current_device()) != DSA_OK) return s;
  void* scratch = nullptr;
  s = scratch_for_current_device(&scratch);
  if (s != DSA_OK) return s;
  s = dsa_prefill_layer(dims, q, latent, rope, q_idx, k_idx, w_idx, out, lse, idx_out, scratch,
                        kNoallocScratchBytes, stream);
  if (s != DSA_OK) return s;
  if (device_status &&
      cudaMemcpyAsync(device_status, scratch, sizeof(uint32_t), cudaMemcpyDeviceToDevice,
                      static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return DSA_ERR_CUDA;
  return DSA_OK;
}
