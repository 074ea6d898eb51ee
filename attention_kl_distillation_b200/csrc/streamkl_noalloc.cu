// streamkl_noalloc.cu -- a backward entry point that allocates nothing.
//
// Some callers cannot allocate device memory when they need the gradient:
// a framework whose caching allocator already owns the free device memory
// (a cudaMalloc from outside it can fail, or fragment its pool), or code that
// must not call cudaMalloc/cudaFree because those calls may synchronise the
// whole device.  streamkl_bwd already allocates nothing, but it asks the
// caller for a workspace.  streamkl_bwd_noalloc instead uses scratch that
// this library owns: one statically sized device array, reserved on a GPU
// when this module is loaded there (at context creation under eager module
// loading, at first use under lazy loading) and kept until the process exits.
#include "streamkl.h"

#include <cuda_runtime.h>

#include <mutex>

namespace {

// The scratch itself.  Host code must not use this name as a device address
// (on the host it is only a stand-in symbol); its device address comes from
// cudaGetSymbolAddress, looked up once per device below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[STREAMKL_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

}  // namespace

extern "C" streamkl_status streamkl_bwd_noalloc(const streamkl_problem* prob, const float* dL,
                                                const void* Q1, const void* K1, const void* Q2,
                                                const void* K2, const float* L, const float* LSE1,
                                                const float* LSE2, void* dQ1, void* dK1,
                                                void* dQ2, void* dK2, streamkl_stream_t stream) {
  const size_t need = streamkl_bwd_workspace_size(prob);
  if (need == 0)  // bad problem: let the ordinary entry point report which error
    return streamkl_bwd(prob, dL, Q1, K1, Q2, K2, L, LSE1, LSE2, dQ1, dK1, dQ2, dK2, nullptr, 0,
                        stream);
  if (need > STREAMKL_NOALLOC_SCRATCH_BYTES) return STREAMKL_EINVAL;

  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return STREAMKL_ECUDA;
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_scratch_addr[dev]) {
      void* addr = nullptr;
      if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || addr == nullptr)
        return STREAMKL_ECUDA;
      g_scratch_addr[dev] = addr;
    }
    scratch = g_scratch_addr[dev];
  }
  // streamkl_bwd clears the parts of its workspace that must start at zero
  // (the dQ accumulator and the work-unit counter) on every call.
  return streamkl_bwd(prob, dL, Q1, K1, Q2, K2, L, LSE1, LSE2, dQ1, dK1, dQ2, dK2, scratch,
                      STREAMKL_NOALLOC_SCRATCH_BYTES, stream);
}

extern "C" size_t streamkl_bwd_noalloc_scratch_bytes(void) {
  return STREAMKL_NOALLOC_SCRATCH_BYTES;
}
