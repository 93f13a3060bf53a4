// m3ssd_bwd_noalloc: the backward with its scratch in a fixed file-scope
// device array instead of a caller-provided workspace.
//
// The array is reserved once, when the library's device code is loaded.
// Requests whose workspace (m3ssd_bwd_workspace_size) exceeds it are refused
// before any device call.  All calls share the one array, so they must not
// run concurrently.
#include <cuda_runtime.h>

#include "../../include/m3ssd.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(64) << 20;  // 64 MiB

static __device__ __align__(256) unsigned char g_bwd_scratch[kStaticScratchBytes];

}  // namespace

extern "C" m3ssd_status m3ssd_bwd_noalloc(const m3ssd_dims* dims, const void* X,
                                          const float* logdecay, const float* beta,
                                          const float* gamma, const void* B, const void* C,
                                          const float* theta, const float* D, const float* h0,
                                          const m3ssd_fwd_extra* extra, const void* dY,
                                          const float* dhT, const m3ssd_bwd_grads* grads,
                                          void* stream) {
  if (!dims) return M3SSD_ERR_INVALID_ARG;
  if (m3ssd_bwd_workspace_size(dims) > kStaticScratchBytes) return M3SSD_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if (cudaGetSymbolAddress(&scratch, g_bwd_scratch) != cudaSuccess) {
    (void)cudaGetLastError();
    return M3SSD_ERR_CUDA;
  }
  return m3ssd_bwd(dims, X, logdecay, beta, gamma, B, C, theta, D, h0, extra, dY, dhT, grads,
                   scratch, kStaticScratchBytes, stream);
}
