// Decode step of the Mamba-3 SISO scan on an fp32 cache.
//
// The step is a pure stream over the (b, H, N, P) fp32 state: every element is
// read once and written once, and SISO decode has O(1) arithmetic per state
// element ("TorchMamba" README, "Math notes", MIMO paragraph: SISO decode
// intensity is Theta(1)).  One CTA owns one (b, h) state (N*P floats), reads it
// with 128-bit loads along P (a warp covers two full 256-byte rows for P = 64),
// updates it in place and reduces y = Cbar^T h across the CTA.
//
//   phi' = angle + theta_t;  Bbar_prev = R(angle) b_prev;  Bbar = R(phi') B_t;
//   Cbar = R(phi') C_t;  h = alpha h + beta Bbar_prev x_prev^T + gamma Bbar x_t^T;
//   y = Cbar^T h + D x_t;  angle = phi' (stored reduced to [-pi, pi]), x_prev = x_t.
// b_prev is per group and shared by H/G heads, so it is replaced by B_t in a
// second, tiny launch once every head has read it.
#include "common.cuh"
#include "internal.h"

namespace m3ssd {
namespace {

constexpr int kThreads = 256;
constexpr int kRowsInFlight = 8;  // state rows a thread loads before it computes

template <int VEC>
struct VecT;
template <>
struct VecT<4> {
  using type = float4;
};
template <>
struct VecT<1> {
  using type = float;
};

__device__ __forceinline__ void ld_vec(const float* p, float (&v)[4]) {
  const float4 t = *reinterpret_cast<const float4*>(p);
  v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
}
__device__ __forceinline__ void st_vec(float* p, const float (&v)[4]) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
__device__ __forceinline__ void ld_vec(const float* p, float (&v)[1]) { v[0] = *p; }
__device__ __forceinline__ void st_vec(float* p, const float (&v)[1]) { *p = v[0]; }

template <typename T, int VEC>
__global__ void __launch_bounds__(kThreads) step_kernel(StepArgs a) {
  extern __shared__ float smem[];
  const int64_t H = a.H, P = a.P, N = a.N, G = a.G;
  const int64_t NH = N / 2;
  const int64_t bh = blockIdx.x;
  const int64_t b = bh / H, h = bh % H, g = h / (H / G);
  const int tid = threadIdx.x;

  float* Bb = smem;       // N   Bbar_t
  float* Cb = Bb + N;     // N   Cbar_t
  float* Bpb = Cb + N;    // N   Bbar_{t-1}
  float* xs = Bpb + N;    // P   x_t
  float* xps = xs + P;    // P   x_{t-1}
  float* red = xps + P;   // R*P partial sums of y

  const T* Bt = static_cast<const T*>(a.B_t) + (b * G + g) * N;
  const T* Ct = static_cast<const T*>(a.C_t) + (b * G + g) * N;
  const float* bprev = a.b_prev + (b * G + g) * N;

  for (int64_t i = tid; i < NH; i += kThreads) {
    const float ang = a.angle[bh * NH + i];
    const float ph = wrap_angle(ang + (a.theta_t ? a.theta_t[bh * NH + i] : 0.f));
    float s, c, s0, c0;
    sincosf(ph, &s, &c);
    sincosf(ang, &s0, &c0);
    float bx = to_f32(Bt[2 * i]), by = to_f32(Bt[2 * i + 1]);
    float cx = to_f32(Ct[2 * i]), cy = to_f32(Ct[2 * i + 1]);
    float px = bprev[2 * i], py = bprev[2 * i + 1];
    if (a.Bbias) {
      const float u0 = a.Bbias[h * N + 2 * i], u1 = a.Bbias[h * N + 2 * i + 1];
      bx += u0; by += u1; px += u0; py += u1;
    }
    if (a.Cbias) {
      cx += a.Cbias[h * N + 2 * i];
      cy += a.Cbias[h * N + 2 * i + 1];
    }
    const float2 rb = rot2(c, s, bx, by);
    const float2 rc = rot2(c, s, cx, cy);
    const float2 rp = rot2(c0, s0, px, py);
    Bb[2 * i] = rb.x; Bb[2 * i + 1] = rb.y;
    Cb[2 * i] = rc.x; Cb[2 * i + 1] = rc.y;
    Bpb[2 * i] = rp.x; Bpb[2 * i + 1] = rp.y;
    a.angle[bh * NH + i] = ph;
  }
  const T* xt = static_cast<const T*>(a.x_t) + bh * P;
  for (int64_t p = tid; p < P; p += kThreads) {
    const float x = to_f32(xt[p]);
    xs[p] = x;
    xps[p] = a.x_prev[bh * P + p];
    a.x_prev[bh * P + p] = x;
  }
  const float alpha = expf(a.logdecay_t[bh]);
  const float be = a.beta_t ? a.beta_t[bh] : 0.f;
  const float ga = a.gamma_t[bh];
  __syncthreads();

  const int QP = (int)P / VEC;       // vectors per state row
  const int R = kThreads / QP;       // rows updated concurrently
  const int q = tid % QP, r0 = tid / QP;
  float* S = a.ssm + bh * N * P;
  float acc[VEC];
#pragma unroll
  for (int j = 0; j < VEC; ++j) acc[j] = 0.f;
  if (r0 < R) {
    float xv[VEC], xpv[VEC];
#pragma unroll
    for (int j = 0; j < VEC; ++j) {
      xv[j] = xs[q * VEC + j];
      xpv[j] = xps[q * VEC + j];
    }
    for (int64_t n0 = r0; n0 < N; n0 += (int64_t)R * kRowsInFlight) {
      float hv[kRowsInFlight][VEC];
#pragma unroll
      for (int k = 0; k < kRowsInFlight; ++k) {
        const int64_t n = n0 + (int64_t)k * R;
        if (n < N) ld_vec(S + n * P + q * VEC, hv[k]);
      }
#pragma unroll
      for (int k = 0; k < kRowsInFlight; ++k) {
        const int64_t n = n0 + (int64_t)k * R;
        if (n < N) {
          const float bp = be * Bpb[n], bc = ga * Bb[n], cc = Cb[n];
#pragma unroll
          for (int j = 0; j < VEC; ++j) {
            const float v = alpha * hv[k][j] + bp * xpv[j] + bc * xv[j];
            hv[k][j] = v;
            acc[j] += cc * v;
          }
          st_vec(S + n * P + q * VEC, hv[k]);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < VEC; ++j) red[r0 * P + q * VEC + j] = acc[j];
  }
  __syncthreads();

  T* yt = static_cast<T*>(a.y_t) + bh * P;
  for (int64_t p = tid; p < P; p += kThreads) {
    float y = a.D ? a.D[h] * xs[p] : 0.f;
    for (int r = 0; r < R; ++r) y += red[r * P + p];
    yt[p] = from_f32<T>(y);
  }
}

// Specialised step for N = 128, P = 64 (the decode workload): 128 threads, each
// owning one 4-wide column slice of 16 state rows.  The 16 float4 loads of the
// state are issued before the rotation prologue, so the state stream (32 KB per
// CTA) is in flight while the angles, sincos and rotations are computed.
constexpr int kN = 128, kP = 64, kThreads128 = 128, kRows = kN / (kThreads128 / (kP / 4));

template <typename T>
__global__ void __launch_bounds__(kThreads128) step_kernel_n128p64(StepArgs a) {
  __shared__ float Bb[kN], Cb[kN], Bpb[kN], xs[kP], xps[kP];
  __shared__ float4 red[kThreads128 / 32][kP / 4];
  const int64_t H = a.H, G = a.G;
  const int64_t bh = blockIdx.x;
  const int64_t b = bh / H, h = bh % H, g = h / (H / G);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int q = tid & 15, r0 = tid >> 4;  // column slice q, rows r0 + 8k
  float4* S = reinterpret_cast<float4*>(a.ssm + bh * kN * kP);
  float4 hv[kRows];
#pragma unroll
  for (int k = 0; k < kRows; ++k) hv[k] = S[(r0 + 8 * k) * (kP / 4) + q];

  const T* Bt = static_cast<const T*>(a.B_t) + (b * G + g) * kN;
  const T* Ct = static_cast<const T*>(a.C_t) + (b * G + g) * kN;
  const float* bprev = a.b_prev + (b * G + g) * kN;
  if (tid < kN / 2) {
    const int i = tid;
    const float ang = a.angle[bh * (kN / 2) + i];
    const float ph = wrap_angle(ang + (a.theta_t ? a.theta_t[bh * (kN / 2) + i] : 0.f));
    float s, c, s0, c0;
    sincosf(ph, &s, &c);
    sincosf(ang, &s0, &c0);
    float bx = to_f32(Bt[2 * i]), by = to_f32(Bt[2 * i + 1]);
    float cx = to_f32(Ct[2 * i]), cy = to_f32(Ct[2 * i + 1]);
    float px = bprev[2 * i], py = bprev[2 * i + 1];
    if (a.Bbias) {
      const float u0 = a.Bbias[h * kN + 2 * i], u1 = a.Bbias[h * kN + 2 * i + 1];
      bx += u0; by += u1; px += u0; py += u1;
    }
    if (a.Cbias) {
      cx += a.Cbias[h * kN + 2 * i];
      cy += a.Cbias[h * kN + 2 * i + 1];
    }
    const float2 rb = rot2(c, s, bx, by);
    const float2 rc = rot2(c, s, cx, cy);
    const float2 rp = rot2(c0, s0, px, py);
    Bb[2 * i] = rb.x; Bb[2 * i + 1] = rb.y;
    Cb[2 * i] = rc.x; Cb[2 * i + 1] = rc.y;
    Bpb[2 * i] = rp.x; Bpb[2 * i + 1] = rp.y;
    a.angle[bh * (kN / 2) + i] = ph;
  } else {
    const int p = tid - kN / 2;
    const float x = to_f32(static_cast<const T*>(a.x_t)[bh * kP + p]);
    xs[p] = x;
    xps[p] = a.x_prev[bh * kP + p];
    a.x_prev[bh * kP + p] = x;
  }
  const float alpha = expf(a.logdecay_t[bh]);
  const float be = a.beta_t ? a.beta_t[bh] : 0.f;
  const float ga = a.gamma_t[bh];
  __syncthreads();

  const float4 xv = reinterpret_cast<const float4*>(xs)[q];
  const float4 xpv = reinterpret_cast<const float4*>(xps)[q];
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int k = 0; k < kRows; ++k) {
    const int n = r0 + 8 * k;
    const float bp = be * Bpb[n], bc = ga * Bb[n], cc = Cb[n];
    float4 v;
    v.x = alpha * hv[k].x + bp * xpv.x + bc * xv.x;
    v.y = alpha * hv[k].y + bp * xpv.y + bc * xv.y;
    v.z = alpha * hv[k].z + bp * xpv.z + bc * xv.z;
    v.w = alpha * hv[k].w + bp * xpv.w + bc * xv.w;
    S[n * (kP / 4) + q] = v;
    acc.x += cc * v.x; acc.y += cc * v.y; acc.z += cc * v.z; acc.w += cc * v.w;
  }
  // lanes l and l + 16 hold the same column slice
  acc.x += __shfl_xor_sync(0xffffffffu, acc.x, 16);
  acc.y += __shfl_xor_sync(0xffffffffu, acc.y, 16);
  acc.z += __shfl_xor_sync(0xffffffffu, acc.z, 16);
  acc.w += __shfl_xor_sync(0xffffffffu, acc.w, 16);
  if (lane < 16) red[warp][q] = acc;
  __syncthreads();
  if (tid < kP) {
    const float* rf = reinterpret_cast<const float*>(red);
    float y = a.D ? a.D[h] * xs[tid] : 0.f;
#pragma unroll
    for (int w = 0; w < kThreads128 / 32; ++w) y += rf[w * kP + tid];
    static_cast<T*>(a.y_t)[bh * kP + tid] = from_f32<T>(y);
  }
}

template <typename T>
__global__ void bprev_update_kernel(const T* __restrict__ B_t, float* __restrict__ b_prev,
                                    int64_t n) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) b_prev[i] = to_f32(B_t[i]);
}

template <typename T, int VEC>
cudaError_t launch_typed(const StepArgs& a, cudaStream_t s) {
  const int QP = (int)a.P / VEC;
  const int R = kThreads / QP;
  const size_t smem = sizeof(float) * (size_t)(3 * a.N + 2 * a.P + (int64_t)R * a.P);
  cudaError_t e = cudaFuncSetAttribute(step_kernel<T, VEC>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  step_kernel<T, VEC><<<(unsigned)(a.b * a.H), kThreads, smem, s>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t nb = a.b * a.G * a.N;
  bprev_update_kernel<T><<<(unsigned)((nb + 255) / 256), 256, 0, s>>>(
      static_cast<const T*>(a.B_t), a.b_prev, nb);
  return cudaGetLastError();
}

}  // namespace

template <typename T>
cudaError_t launch_n128p64(const StepArgs& a, cudaStream_t s) {
  step_kernel_n128p64<T><<<(unsigned)(a.b * a.H), kThreads128, 0, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t nb = a.b * a.G * a.N;
  bprev_update_kernel<T><<<(unsigned)((nb + 255) / 256), 256, 0, s>>>(
      static_cast<const T*>(a.B_t), a.b_prev, nb);
  return cudaGetLastError();
}

cudaError_t launch_step(const StepArgs& a, cudaStream_t s) {
  if (a.b * a.H == 0) return cudaSuccess;
  if (a.N == kN && a.P == kP && (reinterpret_cast<uintptr_t>(a.ssm) % 16 == 0))
    return a.bf16 ? launch_n128p64<__nv_bfloat16>(a, s) : launch_n128p64<float>(a, s);
  const bool vec4 = (a.P % 4 == 0) && (reinterpret_cast<uintptr_t>(a.ssm) % 16 == 0) &&
                    (a.P / 4 <= kThreads);
  if (a.bf16)
    return vec4 ? launch_typed<__nv_bfloat16, 4>(a, s) : launch_typed<__nv_bfloat16, 1>(a, s);
  return vec4 ? launch_typed<float, 4>(a, s) : launch_typed<float, 1>(a, s);
}

}  // namespace m3ssd
