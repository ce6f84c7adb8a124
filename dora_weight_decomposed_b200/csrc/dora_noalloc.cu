// dora_norm_noalloc: the norm call for callers that cannot allocate device
// memory or hand the library a workspace.
//
// Who needs it: a host application whose memory manager has already claimed
// the device memory it is allowed to use (a cudaMalloc would fail or break its
// budget), code that must not trigger cudaMalloc's implicit device
// synchronisation in a latency-critical loop, and thin C bindings that only
// hold the layer's tensors and have no allocator to size and own a workspace.
//
// Instead of a caller-supplied workspace, this call uses the file-scope device
// array below (16 MiB, 256-byte aligned). Every GPU that loads this library
// module keeps that array until the process exits. The first call on a device
// looks up the array's device address (cudaGetSymbolAddress, with that device
// current) and caches it; later calls on that device only read the cache.
// Beyond that look-up it runs exactly the kernels of dora_norm, which write
// every scratch byte they read, so nothing needs clearing between calls. All
// calls on a device share the one array: two calls whose kernels overlap on
// the GPU (different streams, no ordering between them) race on it.
#include <mutex>
#include <string>

#include "dora_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB

// Host code must not use this name as a device address: it is a host-side
// stand-in. The device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_dev[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up once per device).
dora_status_t scratch_for_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return dora::cuda_status(e, "dora_norm_noalloc: cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) {
    dora::set_error("dora_norm_noalloc: device index above 63");
    return DORA_EUNSUPPORTED;
  }
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_dev[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) {
      return dora::cuda_status(e != cudaSuccess ? e : cudaErrorInvalidSymbol,
                               "dora_norm_noalloc: cudaGetSymbolAddress of the scratch array");
    }
    g_scratch_dev[dev] = p;
  }
  *out = g_scratch_dev[dev];
  return DORA_OK;
}

}  // namespace

extern "C" {

dora_status_t dora_norm_noalloc(const dora_desc_t* desc, const void* W0, const void* A, const void* B,
                                const float* m, float* norm_out, float* g_out, float* gm1_out,
                                dora_stream_t stream) {
  const size_t need = dora_workspace_size(desc, 0, DORA_OP_NORM);
  if (need == 0) {
    // Invalid descriptor: let dora_norm report exactly what is wrong.
    return dora_norm(desc, W0, A, B, m, norm_out, g_out, gm1_out, nullptr, 0, stream);
  }
  if (need > kNoAllocScratchBytes) {
    dora::set_error("dora_norm_noalloc: this layer needs " + std::to_string(need) +
                    " bytes of scratch but the built-in scratch array holds " +
                    std::to_string(kNoAllocScratchBytes) + " bytes (16 MiB); use dora_norm with a workspace");
    return DORA_EUNSUPPORTED;
  }
  void* scratch = nullptr;
  const dora_status_t s = scratch_for_current_device(&scratch);
  if (s != DORA_OK) return s;
  return dora_norm(desc, W0, A, B, m, norm_out, g_out, gm1_out, scratch, kNoAllocScratchBytes, stream);
}

}  // extern "C"
