// fa_noalloc.cu -- fa_bwd for callers that cannot allocate device memory.
//
// fa_bwd needs a scratch workspace (the fp32 dQ accumulator, the per-row
// terms D_i and log2-scaled LSE, and the work counter of its scheduler) that
// the caller normally allocates.  Some callers cannot do that: a runtime
// whose device memory is entirely handed out up front by its own pool, so a
// further cudaMalloc would fail or fragment it, or a latency-critical loop in
// which cudaMalloc/cudaFree would stall on an implicit device
// synchronisation.  fa_bwd_static_workspace() serves them: its scratch is a
// fixed array in the library's own device memory, which exists on every GPU
// that loads the library for as long as the process lives.
//
// The array's name is only a host-side stand-in in host code, not a device
// address: the real address is looked up once per device with
// cudaGetSymbolAddress (with that device current) and handed to the kernels.
#include <mutex>

#include "fa.h"
#include "fa_internal.h"

namespace fa {

static __device__ __align__(256) unsigned char g_bwd_static_workspace[FA_BWD_STATIC_WORKSPACE_BYTES];

// Device address of this device's copy of the array, looked up on first use.
static void* static_workspace_ptr() {
  static void* addr[64] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_bwd_static_workspace) != cudaSuccess) return nullptr;
    addr[dev] = p;
  }
  return addr[dev];
}

}  // namespace fa

extern "C" fa_status fa_bwd_static_workspace(const void* Q, const void* K, const void* V, const void* O,
                                             const void* dO, const float* LSE, int B, int H, int N, int d,
                                             int mask_kind, const uint8_t* block_mask, float scale, void* dQ,
                                             void* dK, void* dV, void* stream) {
  // Refuse, before touching the GPU, a problem whose scratch does not fit.
  const size_t need = fa_bwd_workspace_size(B, H, N, d);
  if (need == 0) return (B <= 0 || H <= 0 || N <= 0) ? FA_ERR_INVALID_ARG : FA_ERR_UNSUPPORTED;
  if (need > (size_t)FA_BWD_STATIC_WORKSPACE_BYTES) return FA_ERR_WORKSPACE;
  void* ws = fa::static_workspace_ptr();
  if (!ws) return FA_ERR_CUDA;
  // Same launches as fa_bwd; its prep stage clears everything in the scratch
  // that must start at zero, so what an earlier call left there is harmless.
  return fa_bwd(Q, K, V, O, dO, LSE, B, H, N, d, mask_kind, block_mask, scale, dQ, dK, dV, ws,
                (size_t)FA_BWD_STATIC_WORKSPACE_BYTES, stream);
}
