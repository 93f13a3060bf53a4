// Small device helpers shared by the kernels of libm3ssd.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace m3ssd {

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// Counter-clockwise rotation of the pair (re, im) by the angle whose cosine
// and sine are (c, s): (c re - s im, s re + c im).
__device__ __forceinline__ float2 rot2(float c, float s, float re, float im) {
  return make_float2(c * re - s * im, s * re + c * im);
}

// x reduced to about [-pi, pi] by subtracting k * 2pi, with 2pi split into its
// nearest fp32 value and the fp32 remainder (Cody-Waite argument reduction);
// valid for |x| up to about 1e5.  Angles are stored reduced so that an fp32
// running angle keeps the absolute precision of a number below pi.
__device__ __forceinline__ float wrap_angle(float x) {
  const float k = rintf(x * 0.159154943091895336f);  // x / (2 pi)
  const float r = fmaf(-k, 6.28318548202514648f, x);  // fp32(2 pi)
  return fmaf(-k, -1.74845553146951720e-07f, r);      // 2 pi - fp32(2 pi)
}

// sin and cos of x for |x| up to about 1e5: the reduced argument goes to the
// hardware approximations (absolute error about 1e-6).
__device__ __forceinline__ void fast_sincos(float x, float* s, float* c) {
  __sincosf(wrap_angle(x), s, c);
}

}  // namespace m3ssd
