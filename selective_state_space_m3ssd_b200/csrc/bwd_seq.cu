// Backward of the Mamba-3 SISO scan (fp32, sequential in time), for every
// shape the sequential forward takes.
//
// The recurrence ("TorchMamba" README, "Math notes", M3 SISO)
//   phi_t = phi_{t-1} + theta_t,  Bbar_t = R(phi_t) B_t,  Cbar_t = R(phi_t) C_t
//   h_t = a_t h_{t-1} + beta_t Bbar_{t-1} x_{t-1}^T + gamma_t Bbar_t x_t^T,  a_t = exp(logdecay_t)
//   y_t = Cbar_t^T h_t + D x_t
// is differentiated in reverse time order.  With g = dL/dh_t (starting from dhT):
//   dCbar_t = h_t dy_t,  g += Cbar_t dy_t^T,  dD += dy_t . x_t,  dx_t += D dy_t
//   dlogdecay_t = a_t <g, h_{t-1}>,  dgamma_t = Bbar_t^T g x_t,  dbeta_t = Bbar_{t-1}^T g x_{t-1}
//   dBbar_t = gamma_t g x_t,  dx_t += gamma_t g^T Bbar_t
//   dBbar_{t-1} += beta_t g x_{t-1},  dx_{t-1} += beta_t g^T Bbar_{t-1},  then g <- a_t g
//   through each rotation: dv = R(phi)^T dvbar, dphi_i += -dvbar_{2i} vbar_{2i+1} + dvbar_{2i+1} vbar_{2i}
//   dtheta_t = sum_{s>=t} dphi_s,  dangle0 = sum_{s>=-1} dphi_s,  dh0 = g after token 0.
//
// One CTA per (b, h).  Pass 1 runs the forward and stores the state and the
// angle every kBlk tokens in the workspace; pass 2 walks the blocks backwards,
// recomputes a block's states into the workspace, and sweeps it in reverse.
// Gradients of the group-shared B, C, bprev0 and of D are written per head (per
// sequence for D) and summed in a fixed order by a second kernel, so the
// result does not depend on scheduling.
#include "common.cuh"
#include "internal.h"

namespace m3ssd {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kBlk = 64;  // tokens between state checkpoints

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Workspace regions (floats), in order.
struct BwdWs {
  size_t chk, blk, dBh, dCh, dbph, dDbh;  // byte offsets
  size_t total;
};
BwdWs bwd_ws_layout(int64_t b, int64_t L, int64_t H, int64_t P, int64_t N) {
  const size_t bh = (size_t)(b * H), NP = (size_t)(N * P), NH = (size_t)(N / 2);
  const size_t nblk = (size_t)((L + kBlk - 1) / kBlk);
  BwdWs w;
  w.chk = 0;
  w.blk = w.chk + align256(bh * nblk * (NP + NH) * sizeof(float));
  w.dBh = w.blk + align256(bh * (size_t)(kBlk + 1) * NP * sizeof(float));
  w.dCh = w.dBh + align256((size_t)(b * L * H * N) * sizeof(float));
  w.dbph = w.dCh + align256((size_t)(b * L * H * N) * sizeof(float));
  w.dDbh = w.dbph + align256(bh * (size_t)N * sizeof(float));
  w.total = w.dDbh + align256(bh * sizeof(float));
  return w;
}

template <typename T>
__device__ __forceinline__ float ldx(const T* p, int64_t i) {
  return to_f32(p[i]);
}

// Pairwise rotation of v (N values, from global memory of type T or fp32) by
// phi into out; threads i < N/2 each take one pair.
template <typename V>
__device__ __forceinline__ void rotate_into(const V* v, const float* phi, int64_t NH, float* out) {
  for (int64_t i = threadIdx.x; i < NH; i += kThreads) {
    float s, c;
    __sincosf(phi[i], &s, &c);
    const float re = to_f32(v[2 * i]), im = to_f32(v[2 * i + 1]);
    out[2 * i] = c * re - s * im;
    out[2 * i + 1] = s * re + c * im;
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads) bwd_seq_kernel(BwdArgs a, BwdWs ws) {
  extern __shared__ float smem[];
  const int64_t H = a.H, P = a.P, N = a.N, G = a.G, L = a.L;
  const int64_t NH = N / 2, NP = N * P;
  const int64_t bh = blockIdx.x;
  const int64_t b = bh / H, h = bh % H, g = h / (H / G);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t nblk = (L + kBlk - 1) / kBlk;
  const T* X = static_cast<const T*>(a.X);
  const T* Bg = static_cast<const T*>(a.B);
  const T* Cg = static_cast<const T*>(a.C);
  const T* dY = static_cast<const T*>(a.dY);

  float* Srun = smem;                       // NP  running state of the recompute
  float* gS = Srun + NP;                    // NP  dL/dh
  float* phiB = gS + NP;                    // (kBlk + 1) NH  phi_{t0-1} .. phi_{t0+kBlk-1}
  float* Bb = phiB + (kBlk + 1) * NH;       // N   Bbar_t
  float* Cb = Bb + N;                       // N   Cbar_t
  float* Bp = Cb + N;                       // N   Bbar_{t-1}
  float* dCb = Bp + N;                      // N   dCbar_t
  float* gx = dCb + N;                      // N   g x_t
  float* gxp = gx + N;                      // N   g x_{t-1}
  float* dBc = gxp + N;                     // N   gradient of B_{t-1} carried to token t-1
  float* xv = dBc + N;                      // P   x_t
  float* xpv = xv + P;                      // P   x_{t-1}
  float* dyv = xpv + P;                     // P   dy_t
  float* dxc = dyv + P;                     // P   gradient of x_{t-1} carried to token t-1
  float* pgb = dxc + P;                     // kWarps P  partial g^T Bbar_t
  float* pgbp = pgb + kWarps * P;           // kWarps P  partial g^T Bbar_{t-1}
  float* dphc = pgbp + kWarps * P;          // NH  gradient of phi_{t-1} carried to token t-1
  float* Rth = dphc + NH;                   // NH  running sum of dphi over later tokens
  float* phir = Rth + NH;                   // NH  running angle of the recompute
  float* red = phir + NH;                   // kWarps + 1  (red[kWarps]: running dD)

  char* wsb = static_cast<char*>(a.workspace);
  float* chk = reinterpret_cast<float*>(wsb + ws.chk) + bh * nblk * (NP + NH);
  float* blk = reinterpret_cast<float*>(wsb + ws.blk) + bh * (int64_t)(kBlk + 1) * NP;
  float* dBh = reinterpret_cast<float*>(wsb + ws.dBh);   // (b,L,H,N)
  float* dCh = reinterpret_cast<float*>(wsb + ws.dCh);   // (b,L,H,N)
  float* dbph = reinterpret_cast<float*>(wsb + ws.dbph); // (b,H,N)
  float* dDbh = reinterpret_cast<float*>(wsb + ws.dDbh); // (b,H)
  const float Dh = a.D ? a.D[h] : 0.f;

  // Bbar_{t-1} = R(phi_{t-1}) B_{t-1} (the cache's bprev0 for t = 0) into Bp
  auto rotate_prev = [&](int64_t t, const float* phi_prev) {
    const int64_t tg = (b * L + t) * G + g;
    if (t > 0) {
      rotate_into(Bg + (tg - G) * N, phi_prev, NH, Bp);
    } else if (a.bprev0) {
      rotate_into(a.bprev0 + (b * G + g) * N, phi_prev, NH, Bp);
    } else {
      for (int64_t n = tid; n < N; n += kThreads) Bp[n] = 0.f;
    }
  };
  auto load_x = [&](int64_t t) {
    const int64_t th = (b * L + t) * H + h;
    for (int64_t p = tid; p < P; p += kThreads) {
      xv[p] = ldx(X, th * P + p);
      xpv[p] = t > 0 ? ldx(X, (th - H) * P + p) : (a.xprev0 ? a.xprev0[bh * P + p] : 0.f);
    }
  };
  // one forward token: phir (phi_{t-1} -> phi_t, copied to phi_out), Srun (h_{t-1} -> h_t)
  auto fwd_token = [&](int64_t t, float* phi_out) {
    const int64_t th = (b * L + t) * H + h, tg = (b * L + t) * G + g;
    rotate_prev(t, phir);
    load_x(t);
    __syncthreads();  // phir read
    for (int64_t i = tid; i < NH; i += kThreads) {
      phir[i] = wrap_angle(phir[i] + (a.theta ? a.theta[th * NH + i] : 0.f));
      if (phi_out) phi_out[i] = phir[i];
    }
    __syncthreads();
    rotate_into(Bg + tg * N, phir, NH, Bb);
    __syncthreads();
    const float at = expf(a.logdecay[th]);
    const float be = a.beta ? a.beta[th] : 0.f, ga = a.gamma[th];
    for (int64_t e = tid; e < NP; e += kThreads) {
      const int64_t n = e / P, p = e - n * P;
      Srun[e] = at * Srun[e] + be * Bp[n] * xpv[p] + ga * Bb[n] * xv[p];
    }
    __syncthreads();
  };

  // ---- pass 1: forward, a checkpoint (h_{t0-1}, phi_{t0-1}) every kBlk tokens ----
  for (int64_t i = tid; i < NH; i += kThreads)
    phir[i] = wrap_angle(a.angle0 ? a.angle0[bh * NH + i] : 0.f);
  for (int64_t e = tid; e < NP; e += kThreads) Srun[e] = a.h0 ? a.h0[bh * NP + e] : 0.f;
  __syncthreads();
  for (int64_t t = 0; t < L; ++t) {
    if (t % kBlk == 0) {
      float* c = chk + (t / kBlk) * (NP + NH);
      for (int64_t e = tid; e < NP; e += kThreads) c[e] = Srun[e];
      for (int64_t i = tid; i < NH; i += kThreads) c[NP + i] = phir[i];
    }
    fwd_token(t, nullptr);
  }

  // ---- pass 2: blocks in reverse; recompute a block's states, then sweep it back ----
  for (int64_t e = tid; e < NP; e += kThreads) gS[e] = a.dhT ? a.dhT[bh * NP + e] : 0.f;
  for (int64_t p = tid; p < P; p += kThreads) dxc[p] = 0.f;
  for (int64_t n = tid; n < N; n += kThreads) dBc[n] = 0.f;
  for (int64_t i = tid; i < NH; i += kThreads) { dphc[i] = 0.f; Rth[i] = 0.f; }
  if (tid == 0) red[kWarps] = 0.f;
  __syncthreads();
  for (int64_t k = nblk - 1; k >= 0; --k) {
    const int64_t t0 = k * kBlk, t1 = (t0 + kBlk < L) ? t0 + kBlk : L;
    const float* c = chk + k * (NP + NH);
    for (int64_t e = tid; e < NP; e += kThreads) Srun[e] = blk[e] = c[e];
    for (int64_t i = tid; i < NH; i += kThreads) phir[i] = phiB[i] = c[NP + i];
    __syncthreads();
    for (int64_t t = t0; t < t1; ++t) {
      fwd_token(t, phiB + (t - t0 + 1) * NH);
      for (int64_t e = tid; e < NP; e += kThreads) blk[(t - t0 + 1) * NP + e] = Srun[e];
    }
    __syncthreads();
    for (int64_t t = t1 - 1; t >= t0; --t) {
      const int64_t j = t - t0 + 1;
      const int64_t th = (b * L + t) * H + h, tg = (b * L + t) * G + g;
      const float* St = blk + j * NP;        // h_t
      const float* Sp = blk + (j - 1) * NP;  // h_{t-1}
      const float* ph = phiB + j * NH;       // phi_t
      const float* php = ph - NH;            // phi_{t-1}
      rotate_into(Bg + tg * N, ph, NH, Bb);
      rotate_into(Cg + tg * N, ph, NH, Cb);
      rotate_prev(t, php);
      load_x(t);
      for (int64_t p = tid; p < P; p += kThreads) dyv[p] = ldx(dY, th * P + p);
      __syncthreads();

      // element pass: warp w takes rows n = w, w + 8, ...; lane l columns p = l, l + 32, ...
      const float at = expf(a.logdecay[th]);
      const float be = a.beta ? a.beta[th] : 0.f, ga = a.gamma[th];
      float da = 0.f;
      float pb[8], pbp[8];  // P <= 256
#pragma unroll
      for (int m = 0; m < 8; ++m) { pb[m] = 0.f; pbp[m] = 0.f; }
      for (int64_t n = warp; n < N; n += kWarps) {
        float rc = 0.f, rx = 0.f, rxp = 0.f;
        const float cn = Cb[n], bn = Bb[n], bpn = Bp[n];
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const int64_t p = lane + 32 * m;
          if (p < P) {
            const float gv = gS[n * P + p] + cn * dyv[p];
            rc += St[n * P + p] * dyv[p];
            da += gv * Sp[n * P + p];
            rx += gv * xv[p];
            rxp += gv * xpv[p];
            pb[m] += gv * bn;
            pbp[m] += gv * bpn;
            gS[n * P + p] = at * gv;
          }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          rc += __shfl_xor_sync(0xffffffffu, rc, o);
          rx += __shfl_xor_sync(0xffffffffu, rx, o);
          rxp += __shfl_xor_sync(0xffffffffu, rxp, o);
        }
        if (lane == 0) { dCb[n] = rc; gx[n] = rx; gxp[n] = rxp; }
      }
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const int64_t p = lane + 32 * m;
        if (p < P) { pgb[warp * P + p] = pb[m]; pgbp[warp * P + p] = pbp[m]; }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) da += __shfl_xor_sync(0xffffffffu, da, o);
      if (lane == 0) red[warp] = da;
      __syncthreads();

      // per column: dx_t and the carry to x_{t-1}
      for (int64_t p = tid; p < P; p += kThreads) {
        float gb = 0.f, gbp = 0.f;
        for (int w = 0; w < kWarps; ++w) { gb += pgb[w * P + p]; gbp += pgbp[w * P + p]; }
        a.dX[th * P + p] = dxc[p] + Dh * dyv[p] + ga * gb;
        dxc[p] = be * gbp;
      }
      // scalars: dgamma, dbeta (warp 0), dD (warp 1), dlogdecay (warp 2)
      if (warp == 0) {
        float sg = 0.f, sb = 0.f;
        for (int64_t n = lane; n < N; n += 32) { sg += Bb[n] * gx[n]; sb += Bp[n] * gxp[n]; }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          sg += __shfl_xor_sync(0xffffffffu, sg, o);
          sb += __shfl_xor_sync(0xffffffffu, sb, o);
        }
        if (lane == 0) {
          a.dgamma[th] = sg;
          if (a.dbeta) a.dbeta[th] = sb;
        }
      } else if (warp == 1) {
        float sd = 0.f;
        for (int64_t p = lane; p < P; p += 32) sd += dyv[p] * xv[p];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sd += __shfl_xor_sync(0xffffffffu, sd, o);
        if (lane == 0) red[kWarps] += sd;
      } else if (warp == 2 && lane == 0) {
        float s = 0.f;
        for (int w = 0; w < kWarps; ++w) s += red[w];
        a.dlogdecay[th] = at * s;
      }
      // through the rotations (pair i): B_t and C_t by phi_t, B_{t-1} by phi_{t-1}
      for (int64_t i = tid; i < NH; i += kThreads) {
        float s, cc;
        __sincosf(ph[i], &s, &cc);
        const float d0 = ga * gx[2 * i], d1 = ga * gx[2 * i + 1];
        const float e0 = dCb[2 * i], e1 = dCb[2 * i + 1];
        dBh[th * N + 2 * i] = cc * d0 + s * d1 + dBc[2 * i];
        dBh[th * N + 2 * i + 1] = -s * d0 + cc * d1 + dBc[2 * i + 1];
        dCh[th * N + 2 * i] = cc * e0 + s * e1;
        dCh[th * N + 2 * i + 1] = -s * e0 + cc * e1;
        const float dphi = -d0 * Bb[2 * i + 1] + d1 * Bb[2 * i] - e0 * Cb[2 * i + 1] +
                           e1 * Cb[2 * i] + dphc[i];
        Rth[i] += dphi;
        if (a.dtheta) a.dtheta[th * NH + i] = Rth[i];
        float sp, cp;
        __sincosf(php[i], &sp, &cp);
        const float f0 = be * gxp[2 * i], f1 = be * gxp[2 * i + 1];
        dBc[2 * i] = cp * f0 + sp * f1;
        dBc[2 * i + 1] = -sp * f0 + cp * f1;
        dphc[i] = -f0 * Bp[2 * i + 1] + f1 * Bp[2 * i];
      }
      __syncthreads();
    }
  }

  // ---- gradients of the initial state and the cache inputs ---------------------
  if (a.dh0)
    for (int64_t e = tid; e < NP; e += kThreads) a.dh0[bh * NP + e] = gS[e];
  if (a.dxprev0)
    for (int64_t p = tid; p < P; p += kThreads) a.dxprev0[bh * P + p] = dxc[p];
  for (int64_t n = tid; n < N; n += kThreads) dbph[bh * N + n] = dBc[n];
  if (a.dangle0)
    for (int64_t i = tid; i < NH; i += kThreads) a.dangle0[bh * NH + i] = Rth[i] + dphc[i];
  if (tid == 0) dDbh[bh] = red[kWarps];
}

// Group sums over the heads of a group (dB, dC, dbprev0) and batch sums (dD),
// each in a fixed order.
__global__ void bwd_reduce_kernel(BwdArgs a, BwdWs ws) {
  const int64_t H = a.H, N = a.N, G = a.G, hpg = H / G;
  const int64_t nBC = a.b * a.L * G * N, nbp = a.b * G * N;
  const char* wsb = static_cast<const char*>(a.workspace);
  const float* dBh = reinterpret_cast<const float*>(wsb + ws.dBh);
  const float* dCh = reinterpret_cast<const float*>(wsb + ws.dCh);
  const float* dbph = reinterpret_cast<const float*>(wsb + ws.dbph);
  const float* dDbh = reinterpret_cast<const float*>(wsb + ws.dDbh);
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < nBC + nbp + H;
       idx += stride) {
    if (idx < nBC) {
      const int64_t n = idx % N, gg = (idx / N) % G, bt = idx / (N * G);
      float sb = 0.f, sc = 0.f;
      for (int64_t k = 0; k < hpg; ++k) {
        sb += dBh[(bt * H + gg * hpg + k) * N + n];
        sc += dCh[(bt * H + gg * hpg + k) * N + n];
      }
      a.dB[idx] = sb;
      a.dC[idx] = sc;
    } else if (idx < nBC + nbp) {
      const int64_t r = idx - nBC;
      const int64_t n = r % N, gg = (r / N) % G, bb = r / (N * G);
      float s = 0.f;
      for (int64_t k = 0; k < hpg; ++k) s += dbph[(bb * H + gg * hpg + k) * N + n];
      if (a.dbprev0) a.dbprev0[r] = s;
    } else {
      const int64_t hh = idx - nBC - nbp;
      float s = 0.f;
      for (int64_t bb = 0; bb < a.b; ++bb) s += dDbh[bb * H + hh];
      if (a.dD) a.dD[hh] = s;
    }
  }
}

size_t smem_bytes(int64_t P, int64_t N) {
  const int64_t NH = N / 2;
  return sizeof(float) * (size_t)(2 * N * P + (kBlk + 1) * NH + 7 * N + 4 * P + 2 * kWarps * P +
                                  3 * NH + kWarps + 1);
}

}  // namespace

size_t bwd_workspace_bytes(int64_t b, int64_t L, int64_t H, int64_t P, int64_t N) {
  return bwd_ws_layout(b, L, H, P, N).total;
}

cudaError_t launch_bwd_seq(const BwdArgs& a, cudaStream_t s) {
  if (a.b * a.H == 0) return cudaSuccess;
  const BwdWs ws = bwd_ws_layout(a.b, a.L, a.H, a.P, a.N);
  const size_t smem = smem_bytes(a.P, a.N);
  cudaError_t e;
  if (a.bf16) {
    e = cudaFuncSetAttribute(bwd_seq_kernel<__nv_bfloat16>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    bwd_seq_kernel<__nv_bfloat16><<<(unsigned)(a.b * a.H), kThreads, smem, s>>>(a, ws);
  } else {
    e = cudaFuncSetAttribute(bwd_seq_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    bwd_seq_kernel<float><<<(unsigned)(a.b * a.H), kThreads, smem, s>>>(a, ws);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t total = a.b * a.L * a.G * a.N + a.b * a.G * a.N + a.H;
  const unsigned grid = (unsigned)((total + 255) / 256 < 4096 ? (total + 255) / 256 : 4096);
  bwd_reduce_kernel<<<grid > 0 ? grid : 1, 256, 0, s>>>(a, ws);
  return cudaGetLastError();
}

}  // namespace m3ssd
