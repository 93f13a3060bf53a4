// m3ssd_bwd_noalloc: the backward with its scratch in a fixed file-scope
// device array instead of a caller-provided workspace, for callers that cannot
// allocate device memory at the point of the call (for example code running
// inside a CUDA graph capture, or a host runtime whose allocator may not be
// called from the thread that launches the work).
//
// The array is reserved once, when the library's device code is loaded on a
// device, and every GPU that loads the library keeps it until the process
// exits.  Host code cannot pass the array's name to a kernel: on the host that
// name is a stand-in, not a device address.  The device address is looked up
// with cudaGetSymbolAddress the first time the entry point runs on a device
// (with that device current) and kept per device; that first call should come
// before any stream capture.  Requests whose workspace (m3ssd_bwd_workspace_size)
// exceeds the array are refused before any device call, and invalid dims are
// reported before the address is looked up.  All calls share the one array and
// it keeps the last call's contents (the backward writes every scratch element
// it reads), so calls that overlap on the GPU race.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/m3ssd.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(64) << 20;  // 64 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_bwd_scratch[kStaticScratchBytes];

// The array's device address, looked up once per device.
void* scratch_address(m3ssd_status* st) {
  static void* addr[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    (void)cudaGetLastError();
    *st = M3SSD_ERR_CUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_bwd_scratch) != cudaSuccess || p == nullptr) {
      (void)cudaGetLastError();
      *st = M3SSD_ERR_CUDA;
      return nullptr;
    }
    addr[dev] = p;
  }
  *st = M3SSD_OK;
  return addr[dev];
}

}  // namespace

extern "C" m3ssd_status m3ssd_bwd_noalloc(const m3ssd_dims* dims, const void* X,
                                          const float* logdecay, const float* beta,
                                          const float* gamma, const void* B, const void* C,
                                          const float* theta, const float* D, const float* h0,
                                          const m3ssd_fwd_extra* extra, const void* dY,
                                          const float* dhT, const m3ssd_bwd_grads* grads,
                                          void* stream) {
  if (!dims) return M3SSD_ERR_INVALID_ARG;
  const size_t need = m3ssd_bwd_workspace_size(dims);
  if (need > kStaticScratchBytes) return M3SSD_ERR_UNSUPPORTED;
  if (need == 0)  // invalid dims (the backward reports them) or no scratch needed
    return m3ssd_bwd(dims, X, logdecay, beta, gamma, B, C, theta, D, h0, extra, dY, dhT, grads,
                     nullptr, 0, stream);
  m3ssd_status st = M3SSD_OK;
  void* scratch = scratch_address(&st);
  if (st != M3SSD_OK) return st;
  return m3ssd_bwd(dims, X, logdecay, beta, gamma, B, C, theta, D, h0, extra, dY, dhT, grads,
                   scratch, kStaticScratchBytes, stream);
}
