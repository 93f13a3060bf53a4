// The optional non-finite check of the scan's outputs (M3SSD_CHECK_FINITE).
//
// With the flag set, m3ssd_fwd and m3ssd_step scan the outputs they just wrote
// (Y and hT, or y_t) on the same stream, after their own kernels: a value that
// is NaN or infinite (from an input that was, or from an intermediate that
// overflowed) sets a device word that m3ssd_nonfinite_outputs reads and clears.
// The pages' Burn implementation carries the same switch ("Crate burn_mamba",
// DENY_NAN / DENY_INF); checking the outputs rather than the inputs reads a
// fifth of the bytes and also catches an overflow inside the scan.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"

namespace m3ssd {

__device__ unsigned int g_nonfinite;

namespace {

// Grid-stride over 16-byte granules (8 bf16 or 4 fp32; vec, 16-byte aligned)
// and then element by element over what is left (everything when !vec).  A
// value is non-finite when its exponent field is all ones.
__global__ void nonfinite_kernel(const void* p, int64_t n, bool bf16, bool vec) {
  bool bad = false;
  const int64_t per = bf16 ? 8 : 4;
  const int64_t ng = vec ? n / per : 0;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t i0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  for (int64_t i = i0; i < ng; i += stride) {
    const uint4 v = __ldcs(reinterpret_cast<const uint4*>(p) + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k)
      bad |= bf16 ? ((w[k] & 0x7f80u) == 0x7f80u || (w[k] & 0x7f800000u) == 0x7f800000u)
                  : (w[k] & 0x7f800000u) == 0x7f800000u;
  }
  for (int64_t i = ng * per + i0; i < n; i += stride) {
    const float x = bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i])
                         : reinterpret_cast<const float*>(p)[i];
    bad |= !isfinite(x);
  }
  if (__syncthreads_or(bad) && threadIdx.x == 0) atomicOr(&g_nonfinite, 1u);
}

}  // namespace

cudaError_t launch_nonfinite_check(const void* p, int64_t n, bool bf16, cudaStream_t s) {
  if (p == nullptr || n <= 0) return cudaSuccess;
  const bool vec = (reinterpret_cast<uintptr_t>(p) & 15) == 0;
  const int64_t work = vec ? n / (bf16 ? 8 : 4) + 1 : n;
  int64_t blocks = (work + 255) / 256;
  if (blocks > 1184) blocks = 1184;  // 148 SMs x 8 CTAs of 256 threads
  nonfinite_kernel<<<(unsigned)blocks, 256, 0, s>>>(p, n, bf16, vec);
  return cudaGetLastError();
}

cudaError_t read_and_clear_nonfinite(unsigned int* flag) {
  const unsigned int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(flag, g_nonfinite, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_nonfinite, &zero, sizeof(unsigned int));
}

}  // namespace m3ssd
