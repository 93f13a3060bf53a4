// Sequential fp32 forward of the Mamba-3 SISO scan.
//
// One CTA walks one (b, h) sequence token by token, exactly in the order of
// the recurrence ("TorchMamba" README, "Math notes", M3 SISO):
//   phi_t = phi_{t-1} + theta_t
//   Bbar_t = R(phi_t) B_t,  Cbar_t = R(phi_t) C_t
//   h_t = alpha_t h_{t-1} + beta_t Bbar_{t-1} x_{t-1}^T + gamma_t Bbar_t x_t^T
//   y_t = Cbar_t^T h_t + D x_t
// The fp32 state lives in shared memory; Bbar_{t-1} is kept from the previous
// token instead of being rotated again; the running angle is kept reduced to
// [-pi, pi].  This path serves fp32 inputs (where
// bf16 tensor-core operands would not meet a 1e-4 relative bound) and every
// shape the chunked tensor-core path does not cover.
#include "common.cuh"
#include "internal.h"

namespace m3ssd {
namespace {

constexpr int kThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kThreads) fwd_seq_kernel(FwdArgs a) {
  extern __shared__ float smem[];
  const int64_t H = a.H, P = a.P, N = a.N, G = a.G, L = a.L;
  const int64_t NH = N / 2;
  const int64_t bh = blockIdx.x;
  const int64_t b = bh / H, h = bh % H, g = h / (H / G);
  const int tid = threadIdx.x;
  const int NG = kThreads / (int)P;  // row groups of the state update

  float* S = smem;                    // N*P state
  float* Bbuf = S + N * P;            // 2*N: Bbar of the current / previous token
  float* Cb = Bbuf + 2 * N;           // N
  float* xbuf = Cb + N;               // 2*P: x of the current / previous token
  float* phi = xbuf + 2 * P;          // NH
  float* red = phi + NH;              // NG*P partial sums of y
  float* coef = red + NG * P;         // alpha, beta, gamma

  const T* X = static_cast<const T*>(a.X);
  const T* Bm = static_cast<const T*>(a.B);
  const T* Cm = static_cast<const T*>(a.C);
  T* Y = static_cast<T*>(a.Y);

  for (int64_t e = tid; e < N * P; e += kThreads) S[e] = a.h0 ? a.h0[bh * N * P + e] : 0.f;
  // buffer 1 holds the "previous token": Bbar_{-1} = R(angle0) bprev0, x_{-1} = xprev0
  for (int64_t i = tid; i < NH; i += kThreads) {
    const float ph = a.angle0 ? a.angle0[bh * NH + i] : 0.f;
    phi[i] = ph;
    float s, c;
    sincosf(ph, &s, &c);
    const float b0 = (a.bprev0 ? a.bprev0[(b * G + g) * N + 2 * i] : 0.f) +
                     (a.Bbias ? a.Bbias[h * N + 2 * i] : 0.f);
    const float b1 = (a.bprev0 ? a.bprev0[(b * G + g) * N + 2 * i + 1] : 0.f) +
                     (a.Bbias ? a.Bbias[h * N + 2 * i + 1] : 0.f);
    const float2 r = rot2(c, s, b0, b1);
    Bbuf[N + 2 * i] = r.x;
    Bbuf[N + 2 * i + 1] = r.y;
  }
  for (int64_t p = tid; p < P; p += kThreads) xbuf[P + p] = a.xprev0 ? a.xprev0[bh * P + p] : 0.f;
  __syncthreads();

  int cur = 0;
  for (int64_t t = 0; t < L; ++t) {
    const int64_t th = (b * L + t) * H + h;
    const int64_t tg = (b * L + t) * G + g;
    float* Bc = Bbuf + cur * N;
    const float* Bp = Bbuf + (cur ^ 1) * N;
    float* xc = xbuf + cur * P;
    const float* xp = xbuf + (cur ^ 1) * P;

    for (int64_t i = tid; i < NH; i += kThreads) {
      const float ph = wrap_angle(phi[i] + (a.theta ? a.theta[th * NH + i] : 0.f));
      phi[i] = ph;
      float s, c;
      sincosf(ph, &s, &c);
      float b0 = to_f32(Bm[tg * N + 2 * i]), b1 = to_f32(Bm[tg * N + 2 * i + 1]);
      float c0 = to_f32(Cm[tg * N + 2 * i]), c1 = to_f32(Cm[tg * N + 2 * i + 1]);
      if (a.Bbias) {
        b0 += a.Bbias[h * N + 2 * i];
        b1 += a.Bbias[h * N + 2 * i + 1];
      }
      if (a.Cbias) {
        c0 += a.Cbias[h * N + 2 * i];
        c1 += a.Cbias[h * N + 2 * i + 1];
      }
      const float2 rb = rot2(c, s, b0, b1);
      const float2 rc = rot2(c, s, c0, c1);
      Bc[2 * i] = rb.x;
      Bc[2 * i + 1] = rb.y;
      Cb[2 * i] = rc.x;
      Cb[2 * i + 1] = rc.y;
    }
    for (int64_t p = tid; p < P; p += kThreads) xc[p] = to_f32(X[th * P + p]);
    if (tid == 0) {
      coef[0] = expf(a.logdecay[th]);
      coef[1] = a.beta ? a.beta[th] : 0.f;
      coef[2] = a.gamma[th];
    }
    __syncthreads();

    const float alpha = coef[0], be = coef[1], ga = coef[2];
    const int p = tid % (int)P, grp = tid / (int)P;
    if (grp < NG) {
      float acc = 0.f;
      const float xpp = xp[p], xcp = xc[p];
      for (int64_t n = grp; n < N; n += NG) {
        const int64_t e = n * P + p;
        const float v = alpha * S[e] + be * Bp[n] * xpp + ga * Bc[n] * xcp;
        S[e] = v;
        acc += Cb[n] * v;
      }
      red[grp * P + p] = acc;
    }
    __syncthreads();

    for (int64_t q = tid; q < P; q += kThreads) {
      float y = a.D ? a.D[h] * xc[q] : 0.f;
      for (int r = 0; r < NG; ++r) y += red[r * P + q];
      Y[th * P + q] = from_f32<T>(y);
    }
    cur ^= 1;
  }
  __syncthreads();

  if (a.hT)
    for (int64_t e = tid; e < N * P; e += kThreads) a.hT[bh * N * P + e] = S[e];
  if (a.angleT)
    for (int64_t i = tid; i < NH; i += kThreads) a.angleT[bh * NH + i] = phi[i];
  if (a.xprevT)
    for (int64_t p = tid; p < P; p += kThreads) a.xprevT[bh * P + p] = xbuf[(cur ^ 1) * P + p];
  if (a.bprevT && h % (H / G) == 0) {
    for (int64_t n = tid; n < N; n += kThreads) {
      float v;
      if (L > 0)
        v = to_f32(Bm[((b * L + L - 1) * G + g) * N + n]);
      else
        v = a.bprev0 ? a.bprev0[(b * G + g) * N + n] : 0.f;
      a.bprevT[(b * G + g) * N + n] = v;
    }
  }
}

}  // namespace

cudaError_t launch_fwd_seq(const FwdArgs& a, cudaStream_t s) {
  if ((a.x_tok_stride != 0 && a.x_tok_stride != a.H * a.P) || a.theta16 != nullptr)
    return cudaErrorInvalidValue;
  const int NG = kThreads / (int)a.P;
  const size_t smem =
      sizeof(float) * (size_t)(a.N * a.P + 3 * a.N + 2 * a.P + a.N / 2 + NG * a.P + 4);
  const unsigned grid = (unsigned)(a.b * a.H);
  if (grid == 0) return cudaSuccess;
  cudaError_t e;
  if (a.bf16) {
    e = cudaFuncSetAttribute(fwd_seq_kernel<__nv_bfloat16>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    fwd_seq_kernel<__nv_bfloat16><<<grid, kThreads, smem, s>>>(a);
  } else {
    e = cudaFuncSetAttribute(fwd_seq_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    fwd_seq_kernel<float><<<grid, kThreads, smem, s>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace m3ssd
