// MIMO rank-R scan and decode step (fp32 state; X, B, C, Y in fp32 or bf16).
//
// "TorchMamba" README, table "Models", row Mamba-3 MIMO: a rank-R matmul update
// on a shared (N, P) state; "Functional cores": mimo_loop with X (B,L,H,P,R)
// -> Y (B,L,H,P,R) and h (B,H,N,P); "Math notes", MIMO.  With B and C carrying
// the rank axis as (b,L,G,N,R) and every rank column rotated by the head's
// angle:
//   h_t = a_t h_{t-1} + beta_t sum_r Bbar_{t-1,r} x_{t-1,r}^T + gamma_t sum_r Bbar_{t,r} x_{t,r}^T
//   y_{t,r} = Cbar_{t,r}^T h_t + D x_{t,r}
// One CTA per (b, h).  Thread (rg, p) with p = tid % P and rg = tid / P updates
// the state column p in rows rg, rg + NG, ... and keeps the R partial outputs of
// that column; the NG row groups' partials are summed through shared memory.
// Per state element a token costs 2R fused multiply-adds for the update and R
// for the output against 8 bytes of state traffic in the decode step, so at
// R <= 8 the step stays bound by HBM.
#include "common.cuh"
#include "internal.h"

namespace m3ssd {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxRank = 8;

constexpr int kVecRank = 4;
// The float4 mapping of token_update_v4 applies.
__host__ __device__ constexpr bool vec_ok(int64_t P, int64_t R) {
  return P % 4 == 0 && R <= kVecRank && 4 * kThreads / P >= 1;
}

// Shared-memory layout of one token (floats).
struct MimoSmem {
  float *Bb, *Cb, *Bpb;  // N*R each: rotated B_t, C_t, B_{t-1}
  float *xv, *xpv;       // P*R each: x_t, x_{t-1}
  float *phi, *phip;     // N/2 each: angle of t and of t-1
  float* red;            // NG*P*R partial outputs
};

__device__ __forceinline__ MimoSmem carve(float* base, int64_t N, int64_t P, int64_t R, int NG) {
  MimoSmem m;
  m.Bb = base;
  m.Cb = m.Bb + N * R;
  m.Bpb = m.Cb + N * R;
  m.xv = m.Bpb + N * R;
  m.xpv = m.xv + P * R;
  m.phi = m.xpv + P * R;
  m.phip = m.phi + N / 2;
  m.red = m.phip + N / 2;
  return m;
}
size_t token_smem_floats(int64_t N, int64_t P, int64_t R, bool vec) {
  // partial outputs: one set per row group of the mapping in use
  const int64_t groups = vec ? 4 * kThreads / P : kThreads / P;
  return (size_t)(3 * N * R + 2 * P * R + N + groups * P * R);
}

// Columns of an (N, R) matrix v (element (n, r) at v[n R + r]) rotated pairwise by phi.
template <typename V>
__device__ __forceinline__ void rotate_cols(const V* v, const float* phi, int64_t N, int64_t R,
                                            float* out) {
  const int64_t NH = N / 2;
  for (int64_t k = threadIdx.x; k < NH * R; k += kThreads) {
    const int64_t i = k / R, r = k - i * R;
    float s, c;
    __sincosf(phi[i], &s, &c);
    const float re = to_f32(v[(2 * i) * R + r]), im = to_f32(v[(2 * i + 1) * R + r]);
    out[(2 * i) * R + r] = c * re - s * im;
    out[(2 * i + 1) * R + r] = s * re + c * im;
  }
}

// The state update and the outputs of one token, once Bb, Cb, Bpb, xv, xpv are in
// shared memory.  S is the (N, P) state (shared or global memory); y receives
// the (P, R) outputs in type T.
template <typename T>
__device__ __forceinline__ void token_update(const MimoSmem& m, float* S, int64_t N, int64_t P,
                                             int64_t R, float a, float be, float ga, float Dh,
                                             T* y) {
  const int NG = kThreads / (int)P;
  const int tid = threadIdx.x;
  const int64_t p = tid % P, rg = tid / P;
  if (rg < NG) {
    float acc[kMaxRank];
#pragma unroll
    for (int r = 0; r < kMaxRank; ++r) acc[r] = 0.f;
    for (int64_t n = rg; n < N; n += NG) {
      float ub = 0.f, ug = 0.f;
#pragma unroll
      for (int r = 0; r < kMaxRank; ++r)
        if (r < R) {
          ub += m.Bpb[n * R + r] * m.xpv[p * R + r];
          ug += m.Bb[n * R + r] * m.xv[p * R + r];
        }
      const float s = a * S[n * P + p] + be * ub + ga * ug;
      S[n * P + p] = s;
#pragma unroll
      for (int r = 0; r < kMaxRank; ++r)
        if (r < R) acc[r] += m.Cb[n * R + r] * s;
    }
#pragma unroll
    for (int r = 0; r < kMaxRank; ++r)
      if (r < R) m.red[(rg * P + p) * R + r] = acc[r];
  }
  __syncthreads();
  for (int64_t k = tid; k < P * R; k += kThreads) {
    float s = 0.f;
    for (int g = 0; g < NG; ++g) s += m.red[(int64_t)g * P * R + k];
    y[k] = from_f32<T>(s + Dh * m.xv[k]);
  }
}

// The same for P % 4 == 0 and R <= 4: thread (rg, cg) owns the four columns
// 4 cg .. 4 cg + 3 in rows rg, rg + NG4, ... (NG4 = 4 kThreads / P row groups),
// moves the state as float4 and keeps its x_t, x_{t-1} values in registers.
template <typename T>
__device__ __forceinline__ void token_update_v4(const MimoSmem& m, float* S, int64_t N, int64_t P,
                                                int64_t R, float a, float be, float ga, float Dh,
                                                T* y) {
  const int CG = (int)(P / 4), NG4 = kThreads / CG;
  const int tid = threadIdx.x;
  const int cg = tid % CG, rg = tid / CG;
  if (rg < NG4) {
    float xr[4][kVecRank], xpr[4][kVecRank], acc[4][kVecRank];
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
      for (int r = 0; r < kVecRank; ++r) {
        const bool on = r < R;
        xr[c][r] = on ? m.xv[(4 * cg + c) * R + r] : 0.f;
        xpr[c][r] = on ? m.xpv[(4 * cg + c) * R + r] : 0.f;
        acc[c][r] = 0.f;
      }
    for (int64_t n = rg; n < N; n += NG4) {
      float bb[kVecRank], bp[kVecRank], cc[kVecRank];
#pragma unroll
      for (int r = 0; r < kVecRank; ++r) {
        const bool on = r < R;
        bb[r] = on ? m.Bb[n * R + r] : 0.f;
        bp[r] = on ? m.Bpb[n * R + r] : 0.f;
        cc[r] = on ? m.Cb[n * R + r] : 0.f;
      }
      float4* sp = reinterpret_cast<float4*>(S + n * P + 4 * cg);
      float4 v = *sp;
      float* vv = reinterpret_cast<float*>(&v);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float ub = 0.f, ug = 0.f;
#pragma unroll
        for (int r = 0; r < kVecRank; ++r) {
          ub = fmaf(bp[r], xpr[c][r], ub);
          ug = fmaf(bb[r], xr[c][r], ug);
        }
        vv[c] = a * vv[c] + be * ub + ga * ug;
#pragma unroll
        for (int r = 0; r < kVecRank; ++r) acc[c][r] = fmaf(cc[r], vv[c], acc[c][r]);
      }
      *sp = v;
    }
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
      for (int r = 0; r < kVecRank; ++r)
        if (r < R) m.red[((int64_t)rg * P + 4 * cg + c) * R + r] = acc[c][r];
  }
  __syncthreads();
  for (int64_t k = tid; k < P * R; k += kThreads) {
    float sum = 0.f;
    for (int g2 = 0; g2 < NG4; ++g2) sum += m.red[(int64_t)g2 * P * R + k];
    y[k] = from_f32<T>(sum + Dh * m.xv[k]);
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads) mimo_fwd_kernel(FwdArgs a, int64_t R, bool vec) {
  extern __shared__ float smem[];
  const int64_t H = a.H, P = a.P, N = a.N, G = a.G, L = a.L, NH = N / 2;
  const int64_t bh = blockIdx.x, b = bh / H, h = bh % H, g = h / (H / G);
  const int NG = kThreads / (int)P;
  const int tid = threadIdx.x;
  float* S = smem;
  const MimoSmem m = carve(S + N * P, N, P, R, NG);
  (void)vec;
  const T* X = static_cast<const T*>(a.X);
  const T* Bg = static_cast<const T*>(a.B);
  const T* Cg = static_cast<const T*>(a.C);
  T* Y = static_cast<T*>(a.Y);
  const float Dh = a.D ? a.D[h] : 0.f;

  for (int64_t i = tid; i < NH; i += kThreads)
    m.phi[i] = wrap_angle(a.angle0 ? a.angle0[bh * NH + i] : 0.f);
  for (int64_t e = tid; e < N * P; e += kThreads) S[e] = a.h0 ? a.h0[bh * N * P + e] : 0.f;
  __syncthreads();
  for (int64_t t = 0; t < L; ++t) {
    const int64_t th = (b * L + t) * H + h, tg = (b * L + t) * G + g;
    for (int64_t k = tid; k < P * R; k += kThreads) {
      m.xv[k] = to_f32(X[th * P * R + k]);
      m.xpv[k] = t > 0 ? to_f32(X[(th - H) * P * R + k]) : (a.xprev0 ? a.xprev0[bh * P * R + k] : 0.f);
    }
    // B_{t-1} by phi_{t-1} (the cache's bprev0 for t = 0)
    if (t > 0) {
      rotate_cols(Bg + (tg - G) * N * R, m.phi, N, R, m.Bpb);
    } else if (a.bprev0) {
      rotate_cols(a.bprev0 + (b * G + g) * N * R, m.phi, N, R, m.Bpb);
    } else {
      for (int64_t k = tid; k < N * R; k += kThreads) m.Bpb[k] = 0.f;
    }
    __syncthreads();
    for (int64_t i = tid; i < NH; i += kThreads)
      m.phi[i] = wrap_angle(m.phi[i] + (a.theta ? a.theta[th * NH + i] : 0.f));
    __syncthreads();
    rotate_cols(Bg + tg * N * R, m.phi, N, R, m.Bb);
    rotate_cols(Cg + tg * N * R, m.phi, N, R, m.Cb);
    __syncthreads();
    if (vec)
      token_update_v4<T>(m, S, N, P, R, expf(a.logdecay[th]), a.beta ? a.beta[th] : 0.f,
                         a.gamma[th], Dh, Y + th * P * R);
    else
      token_update<T>(m, S, N, P, R, expf(a.logdecay[th]), a.beta ? a.beta[th] : 0.f,
                      a.gamma[th], Dh, Y + th * P * R);
    __syncthreads();
  }
  if (a.hT)
    for (int64_t e = tid; e < N * P; e += kThreads) a.hT[bh * N * P + e] = S[e];
  if (a.angleT)
    for (int64_t i = tid; i < NH; i += kThreads) a.angleT[bh * NH + i] = m.phi[i];
  if (a.xprevT && L > 0)
    for (int64_t k = tid; k < P * R; k += kThreads)
      a.xprevT[bh * P * R + k] = to_f32(X[((b * L + L - 1) * H + h) * P * R + k]);
  if (a.bprevT && L > 0 && h % (H / G) == 0)
    for (int64_t k = tid; k < N * R; k += kThreads)
      a.bprevT[(b * G + g) * N * R + k] = to_f32(Bg[((b * L + L - 1) * G + g) * N * R + k]);
}

template <typename T>
__global__ void __launch_bounds__(kThreads) mimo_step_kernel(StepArgs a, int64_t R, bool vec) {
  extern __shared__ float smem[];
  const int64_t H = a.H, P = a.P, N = a.N, G = a.G, NH = N / 2;
  const int64_t bh = blockIdx.x, b = bh / H, h = bh % H, g = h / (H / G);
  const int NG = kThreads / (int)P;
  const int tid = threadIdx.x;
  const MimoSmem m = carve(smem, N, P, R, NG);
  const T* x = static_cast<const T*>(a.x_t) + bh * P * R;
  for (int64_t k = tid; k < P * R; k += kThreads) {
    m.xv[k] = to_f32(x[k]);
    m.xpv[k] = a.x_prev[bh * P * R + k];
  }
  for (int64_t i = tid; i < NH; i += kThreads) m.phip[i] = a.angle[bh * NH + i];
  __syncthreads();
  rotate_cols(a.b_prev + (b * G + g) * N * R, m.phip, N, R, m.Bpb);
  for (int64_t i = tid; i < NH; i += kThreads)
    m.phi[i] = wrap_angle(m.phip[i] + (a.theta_t ? a.theta_t[bh * NH + i] : 0.f));
  __syncthreads();
  rotate_cols(static_cast<const T*>(a.B_t) + (b * G + g) * N * R, m.phi, N, R, m.Bb);
  rotate_cols(static_cast<const T*>(a.C_t) + (b * G + g) * N * R, m.phi, N, R, m.Cb);
  __syncthreads();
  if (vec)
    token_update_v4<T>(m, a.ssm + bh * N * P, N, P, R, expf(a.logdecay_t[bh]),
                       a.beta_t ? a.beta_t[bh] : 0.f, a.gamma_t[bh], a.D ? a.D[h] : 0.f,
                       static_cast<T*>(a.y_t) + bh * P * R);
  else
    token_update<T>(m, a.ssm + bh * N * P, N, P, R, expf(a.logdecay_t[bh]),
                    a.beta_t ? a.beta_t[bh] : 0.f, a.gamma_t[bh], a.D ? a.D[h] : 0.f,
                    static_cast<T*>(a.y_t) + bh * P * R);
  for (int64_t i = tid; i < NH; i += kThreads) a.angle[bh * NH + i] = m.phi[i];
  for (int64_t k = tid; k < P * R; k += kThreads) a.x_prev[bh * P * R + k] = m.xv[k];
}

// Specialised decode step for N = 128, P = 64 and R <= 4: 128 threads, thread
// (r0, q) with q = tid % 16 and r0 = tid / 16 owning the 4-wide column slice q
// of rows r0, r0 + 8, ...  Each thread starts the asynchronous copies of its own
// 16 state float4 into shared memory before the rotation prologue, so the
// state stream (32 KB per CTA) is in flight while the angles, sincos and
// rotations are computed; it later reads back only what it copied itself.
constexpr int kMN = 128, kMP = 64, kMThreads = 128, kMRows = kMN / (kMThreads / (kMP / 4));

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst))),
               "l"(gmem_src)
               : "memory");
}

template <typename T, int R>
__global__ void __launch_bounds__(kMThreads) mimo_step_n128p64(StepArgs a) {
  __shared__ float4 Sv[kMN * kMP / 4];
  __shared__ __align__(16) float Bb[kMN * R], Cb[kMN * R], Bpb[kMN * R];
  __shared__ __align__(16) float xs[kMP * R], xps[kMP * R];
  __shared__ __align__(16) float red[kMThreads / 32][kMP * R];
  const int64_t H = a.H, G = a.G;
  const int64_t bh = blockIdx.x, b = bh / H, h = bh % H, g = h / (H / G);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int q = tid & 15, r0 = tid >> 4;
  float4* S = reinterpret_cast<float4*>(a.ssm + bh * kMN * kMP);
#pragma unroll
  for (int k = 0; k < kMRows; ++k) {
    const int e = (r0 + 8 * k) * (kMP / 4) + q;
    cp_async16(&Sv[e], &S[e]);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");

  const int64_t gbase = (b * G + g) * kMN * R;
  if (tid < kMN / 2) {
    const int i = tid;
    const float ang = a.angle[bh * (kMN / 2) + i];
    const float ph = wrap_angle(ang + (a.theta_t ? a.theta_t[bh * (kMN / 2) + i] : 0.f));
    float s, c, s0, c0;
    sincosf(ph, &s, &c);
    sincosf(ang, &s0, &c0);
    const T* Bt = static_cast<const T*>(a.B_t) + gbase;
    const T* Ct = static_cast<const T*>(a.C_t) + gbase;
    const float* bp = a.b_prev + gbase;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int e0 = (2 * i) * R + r, e1 = (2 * i + 1) * R + r;
      const float b0 = to_f32(Bt[e0]), b1 = to_f32(Bt[e1]);
      const float c0v = to_f32(Ct[e0]), c1v = to_f32(Ct[e1]);
      const float p0 = bp[e0], p1 = bp[e1];
      Bb[e0] = c * b0 - s * b1;
      Bb[e1] = s * b0 + c * b1;
      Cb[e0] = c * c0v - s * c1v;
      Cb[e1] = s * c0v + c * c1v;
      Bpb[e0] = c0 * p0 - s0 * p1;
      Bpb[e1] = s0 * p0 + c0 * p1;
    }
    a.angle[bh * (kMN / 2) + i] = ph;
  } else {
    const int p = tid - kMN / 2;
    const T* xt = static_cast<const T*>(a.x_t) + bh * kMP * R;
    float* xp = a.x_prev + bh * kMP * R;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const float x = to_f32(xt[p * R + r]);
      xs[p * R + r] = x;
      xps[p * R + r] = xp[p * R + r];
      xp[p * R + r] = x;
    }
  }
  const float alpha = expf(a.logdecay_t[bh]);
  const float be = a.beta_t ? a.beta_t[bh] : 0.f;
  const float ga = a.gamma_t[bh];
  __syncthreads();

  float acc[4][R];
  if constexpr (R % 2 == 0) {
    // packed fp32 pairs over the rank index r (two FMAs an instruction)
    constexpr int R2 = R / 2;
    float2 xr[4][R2], xpr[4][R2], ac2[4][R2];
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
      for (int j = 0; j < R2; ++j) {
        const int e = (4 * q + c) * R + 2 * j;
        xr[c][j] = make_float2(ga * xs[e], ga * xs[e + 1]);
        xpr[c][j] = make_float2(be * xps[e], be * xps[e + 1]);
        ac2[c][j] = make_float2(0.f, 0.f);
      }
    asm volatile("cp.async.wait_all;" ::: "memory");
#pragma unroll 4
    for (int k = 0; k < kMRows; ++k) {
      const int n = r0 + 8 * k;
      float4 v = Sv[n * (kMP / 4) + q];
      float* vv = reinterpret_cast<float*>(&v);
      float2 bpv[R2], bv[R2], cv[R2];
#pragma unroll
      for (int j = 0; j < R2; ++j) {
        bpv[j] = *reinterpret_cast<const float2*>(&Bpb[n * R + 2 * j]);
        bv[j] = *reinterpret_cast<const float2*>(&Bb[n * R + 2 * j]);
        cv[j] = *reinterpret_cast<const float2*>(&Cb[n * R + 2 * j]);
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float2 s2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < R2; ++j) {
          s2 = __ffma2_rn(bpv[j], xpr[c][j], s2);
          s2 = __ffma2_rn(bv[j], xr[c][j], s2);
        }
        const float u = fmaf(alpha, vv[c], s2.x + s2.y);
        vv[c] = u;
        const float2 u2 = make_float2(u, u);
#pragma unroll
        for (int j = 0; j < R2; ++j) ac2[c][j] = __ffma2_rn(cv[j], u2, ac2[c][j]);
      }
      S[n * (kMP / 4) + q] = v;
    }
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
      for (int j = 0; j < R2; ++j) {
        acc[c][2 * j] = ac2[c][j].x;
        acc[c][2 * j + 1] = ac2[c][j].y;
      }
  } else {
    float xr[4][R], xpr[4][R];
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
      for (int r = 0; r < R; ++r) {
        xr[c][r] = ga * xs[(4 * q + c) * R + r];
        xpr[c][r] = be * xps[(4 * q + c) * R + r];
        acc[c][r] = 0.f;
      }
    asm volatile("cp.async.wait_all;" ::: "memory");
#pragma unroll 4
    for (int k = 0; k < kMRows; ++k) {
      const int n = r0 + 8 * k;
      float4 v = Sv[n * (kMP / 4) + q];
      float* vv = reinterpret_cast<float*>(&v);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float u = alpha * vv[c];
#pragma unroll
        for (int r = 0; r < R; ++r) {
          u = fmaf(Bpb[n * R + r], xpr[c][r], u);
          u = fmaf(Bb[n * R + r], xr[c][r], u);
        }
        vv[c] = u;
#pragma unroll
        for (int r = 0; r < R; ++r) acc[c][r] = fmaf(Cb[n * R + r], u, acc[c][r]);
      }
      S[n * (kMP / 4) + q] = v;
    }
  }
  // lanes l and l + 16 hold the same column slice
#pragma unroll
  for (int c = 0; c < 4; ++c)
#pragma unroll
    for (int r = 0; r < R; ++r) {
      acc[c][r] += __shfl_xor_sync(0xffffffffu, acc[c][r], 16);
      if (lane < 16) red[warp][(4 * q + c) * R + r] = acc[c][r];
    }
  __syncthreads();
  T* yt = static_cast<T*>(a.y_t) + bh * kMP * R;
  const float Dh = a.D ? a.D[h] : 0.f;
  for (int k = tid; k < kMP * R; k += kMThreads) {
    float y = Dh * xs[k];
#pragma unroll
    for (int w = 0; w < kMThreads / 32; ++w) y += red[w][k];
    yt[k] = from_f32<T>(y);
  }
}

// b_prev <- B_t once every head of the step has read the old value.
template <typename T>
__global__ void mimo_bprev_kernel(const T* B_t, float* b_prev, int64_t n) {
  for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < n;
       k += (int64_t)gridDim.x * blockDim.x)
    b_prev[k] = to_f32(B_t[k]);
}

}  // namespace

bool mimo_shape_ok(int64_t N, int64_t P, int64_t R) {
  return R >= 1 && R <= kMaxRank && P <= kThreads && N <= 256 && N * P <= 16384 &&
         sizeof(float) * ((size_t)(N * P) + token_smem_floats(N, P, R, vec_ok(P, R))) <=
             200 * 1024 &&
         sizeof(float) * token_smem_floats(N, P, R, false) <= 48 * 1024;
}

cudaError_t launch_mimo_fwd(const FwdArgs& a, int64_t R, cudaStream_t s) {
  if (a.b * a.H == 0) return cudaSuccess;
  // N = 128, P = 64: the chunked tensor-core kernels, bf16 or fp32 (rank 1 has the
  // SISO layout and runs the SISO ones)
  if (R == 1 && fwd_chunk_supported(a)) return launch_fwd_chunk(a, s);
  if (R == 1 && fwd_chunk32_supported(a)) return launch_fwd_chunk32(a, s);
  if (fwd_chunk_mimo_supported(a, R)) return launch_fwd_chunk_mimo(a, R, s);
  if (fwd_chunk_mimo32_supported(a, R)) return launch_fwd_chunk_mimo32(a, R, s);
  const bool vec = vec_ok(a.P, R);  // the state is in shared memory (16-byte aligned)
  const size_t smem = sizeof(float) * ((size_t)(a.N * a.P) + token_smem_floats(a.N, a.P, R, vec));
  cudaError_t e;
  if (a.bf16) {
    e = cudaFuncSetAttribute(mimo_fwd_kernel<__nv_bfloat16>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    mimo_fwd_kernel<__nv_bfloat16><<<(unsigned)(a.b * a.H), kThreads, smem, s>>>(a, R, vec);
  } else {
    e = cudaFuncSetAttribute(mimo_fwd_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    mimo_fwd_kernel<float><<<(unsigned)(a.b * a.H), kThreads, smem, s>>>(a, R, vec);
  }
  return cudaGetLastError();
}

cudaError_t launch_mimo_step(const StepArgs& a, int64_t R, cudaStream_t s) {
  if (a.b * a.H == 0) return cudaSuccess;
  // float4 state accesses need a 16-byte aligned cache state
  const bool vec = vec_ok(a.P, R) && (reinterpret_cast<uintptr_t>(a.ssm) & 15) == 0;
  const size_t smem = sizeof(float) * token_smem_floats(a.N, a.P, R, vec);
  const int64_t nbp = a.b * a.G * a.N * R;
  const unsigned gbp = (unsigned)((nbp + 255) / 256 < 1024 ? (nbp + 255) / 256 : 1024);
  if (vec && a.N == kMN && a.P == kMP) {
    const unsigned grid = (unsigned)(a.b * a.H);
    if (a.bf16) {
      switch (R) {
        case 1: mimo_step_n128p64<__nv_bfloat16, 1><<<grid, kMThreads, 0, s>>>(a); break;
        case 2: mimo_step_n128p64<__nv_bfloat16, 2><<<grid, kMThreads, 0, s>>>(a); break;
        case 3: mimo_step_n128p64<__nv_bfloat16, 3><<<grid, kMThreads, 0, s>>>(a); break;
        default: mimo_step_n128p64<__nv_bfloat16, 4><<<grid, kMThreads, 0, s>>>(a); break;
      }
      mimo_bprev_kernel<<<gbp, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(a.B_t), a.b_prev, nbp);
    } else {
      switch (R) {
        case 1: mimo_step_n128p64<float, 1><<<grid, kMThreads, 0, s>>>(a); break;
        case 2: mimo_step_n128p64<float, 2><<<grid, kMThreads, 0, s>>>(a); break;
        case 3: mimo_step_n128p64<float, 3><<<grid, kMThreads, 0, s>>>(a); break;
        default: mimo_step_n128p64<float, 4><<<grid, kMThreads, 0, s>>>(a); break;
      }
      mimo_bprev_kernel<<<gbp, 256, 0, s>>>(static_cast<const float*>(a.B_t), a.b_prev, nbp);
    }
    return cudaGetLastError();
  }
  if (a.bf16) {
    mimo_step_kernel<__nv_bfloat16><<<(unsigned)(a.b * a.H), kThreads, smem, s>>>(a, R, vec);
    mimo_bprev_kernel<<<gbp, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(a.B_t), a.b_prev, nbp);
  } else {
    mimo_step_kernel<float><<<(unsigned)(a.b * a.H), kThreads, smem, s>>>(a, R, vec);
    mimo_bprev_kernel<<<gbp, 256, 0, s>>>(static_cast<const float*>(a.B_t), a.b_prev, nbp);
  }
  return cudaGetLastError();
}

}  // namespace m3ssd
