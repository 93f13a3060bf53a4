// Backward of the Mamba-3 SISO scan with the state's columns split across
// CTAs, for N = 128 and P a multiple of 16 (the chunked forward's shape).
//
// The recurrence and its adjoint are those of the sequential backward
// ("TorchMamba" README, "Math notes", M3 SISO):
//   h_t = a_t h_{t-1} + beta_t Bbar_{t-1} x_{t-1}^T + gamma_t Bbar_t x_t^T,  y_t = Cbar_t^T h_t + D x_t
// and, with g = dL/dh_t, token by token in reverse:
//   dCbar_t = h_t dy_t, g += Cbar_t dy_t^T, dlogdecay_t = a_t <g, h_{t-1}>,
//   dgamma_t = Bbar_t^T g x_t, dbeta_t = Bbar_{t-1}^T g x_{t-1},
//   dx_t = D dy_t + gamma_t g^T Bbar_t (+ beta_{t+1} g^T Bbar_t from the next token),
//   dBbar_t = gamma_t g x_t (+ beta_{t+1} g_{t+1} x_t), then g <- a_t g,
// the rotation adjoints dv = R(phi)^T dvbar, dphi_i = -dvbar_{2i} vbar_{2i+1} +
// dvbar_{2i+1} vbar_{2i}, and dtheta_t = sum_{s >= t} dphi_s.
//
// The P columns of the state evolve independently and every quantity that
// mixes them (dCbar, g x, g x_prev, <g, h_{t-1}>, y . x and everything derived
// from them: dB, dC, dtheta, dlogdecay, dgamma, dbeta, dD, dbprev0, dangle0) is a
// sum over columns.  So one CTA takes one (b, h) and one slice of kPS = 16
// columns; thread n owns state row n, keeping its 16 entries of h and of g in
// registers; the per-slice partial sums go to the workspace and a second kernel
// adds the slices (and the heads of a group, and the batch for dD) in a fixed
// order, so the result does not depend on scheduling.  dX, dh0 and dxprev0 are
// per column and written directly.
//
// Pass 1 runs the forward and checkpoints the state slice and the angle every
// kK tokens.  Pass 2 walks the blocks in reverse: it recomputes a block's
// states into the workspace, then sweeps the block back, four CTA barriers a
// token.
#include "common.cuh"
#include "internal.h"

namespace m3ssd {
namespace {

constexpr int kN = 128, kNH = kN / 2, kPS = 16, kT = kN, kK = 16;
constexpr int kPad = kPS + 1;  // row stride of the shared copy of g (no bank conflicts)

size_t al256(size_t x) { return (x + 255) & ~size_t(255); }

struct SplitWs {
  size_t chk, blk, dBp, dCp, dThp, dScal, dbpp, dAngp, dDp, total;
};

SplitWs split_ws_layout(int64_t b, int64_t L, int64_t H, int64_t P) {
  const size_t S = (size_t)(P / kPS), units = (size_t)(b * H) * S;
  const size_t nblk = (size_t)((L + kK - 1) / kK), th = (size_t)(b * L * H), bh = (size_t)(b * H);
  SplitWs w{};
  size_t o = 0;
  auto take = [&](size_t floats) {
    const size_t r = o;
    o += al256(floats * sizeof(float));
    return r;
  };
  w.chk = take(units * nblk * (kN * kPS + kNH));
  w.blk = take(units * (kK + 1) * kN * kPS);
  w.dBp = take(S * th * kN);
  w.dCp = take(S * th * kN);
  w.dThp = take(S * th * kNH);
  w.dScal = take(S * th * 3);
  w.dbpp = take(S * bh * kN);
  w.dAngp = take(S * bh * kNH);
  w.dDp = take(S * bh);
  w.total = o;
  return w;
}

template <typename T>
__device__ __forceinline__ float ld(const T* p, int64_t i) {
  return to_f32(p[i]);
}

template <typename T>
__global__ void __launch_bounds__(kT, 4) bwd_split_kernel(BwdArgs a, SplitWs ws) {
  __shared__ float Bb[3][kN];     // Bbar of tokens, three-deep so one barrier a token suffices
  __shared__ __align__(16) float xs[3][kPS];    // x slices, likewise
  __shared__ float Cb[kN], Bpb[kN], rcv[kN], rxv[kN], rxpv[kN];
  __shared__ __align__(16) float xv[kPS];
  __shared__ __align__(16) float xpv[kPS];
  __shared__ __align__(16) float dyv[kPS];
  __shared__ float gvS[kN * kPad];
  __shared__ float phiB[(kK + 1) * kNH];
  __shared__ float colp[4][2][kPS];
  __shared__ float red[3][kT / 32];  // per warp: <g, h_{t-1}>, Bbar_t . g x_t, Bbar_{t-1} . g x_{t-1}

  const int64_t H = a.H, P = a.P, G = a.G, L = a.L;
  const int S = (int)(P / kPS);
  const int s = blockIdx.x % S;
  const int64_t bh = blockIdx.x / S;
  const int64_t b = bh / H, h = bh % H, g = h / (H / G);
  const int64_t p0 = (int64_t)s * kPS;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = tid;                 // state row of this thread
  const int ri = tid - kNH;          // rotation pair of threads kNH .. kN-1
  const bool rot = tid >= kNH;
  const int64_t nblk = (L + kK - 1) / kK;
  const T* X = static_cast<const T*>(a.X);
  const T* Bg = static_cast<const T*>(a.B);
  const T* Cg = static_cast<const T*>(a.C);
  const T* dY = static_cast<const T*>(a.dY);
  const float Dh = a.D ? a.D[h] : 0.f;

  char* wsb = static_cast<char*>(a.workspace);
  const int64_t unit = bh * S + s;
  float* chk = reinterpret_cast<float*>(wsb + ws.chk) + unit * nblk * (kN * kPS + kNH);
  float* blk = reinterpret_cast<float*>(wsb + ws.blk) + unit * (int64_t)(kK + 1) * kN * kPS;
  const int64_t thN = (int64_t)(a.b * L * H);
  float* dBp = reinterpret_cast<float*>(wsb + ws.dBp) + (int64_t)s * thN * kN;
  float* dCp = reinterpret_cast<float*>(wsb + ws.dCp) + (int64_t)s * thN * kN;
  float* dThp = reinterpret_cast<float*>(wsb + ws.dThp) + (int64_t)s * thN * kNH;
  float* dScal = reinterpret_cast<float*>(wsb + ws.dScal) + (int64_t)s * thN * 3;
  const int64_t bhN = (int64_t)(a.b * H);
  float* dbpp = reinterpret_cast<float*>(wsb + ws.dbpp) + (int64_t)s * bhN * kN;
  float* dAngp = reinterpret_cast<float*>(wsb + ws.dAngp) + (int64_t)s * bhN * kNH;
  float* dDp = reinterpret_cast<float*>(wsb + ws.dDp) + (int64_t)s * bhN;

  // x_{t} slice (t = -1: the cache's xprev0) into buf
  auto load_x = [&](int64_t t, float* buf) {
    if (tid < kPS) {
      if (t >= 0)
        buf[tid] = ld(X, ((b * L + t) * H + h) * P + p0 + tid);
      else
        buf[tid] = a.xprev0 ? a.xprev0[bh * P + p0 + tid] : 0.f;
    }
  };
  // Bbar_t pair ri rotated by phi (t = -1: the cache's bprev0) into buf
  auto rot_B = [&](int64_t t, float phi, float* buf) {
    float re = 0.f, im = 0.f;
    if (t >= 0) {
      const int64_t o = ((b * L + t) * G + g) * kN;
      re = ld(Bg, o + 2 * ri);
      im = ld(Bg, o + 2 * ri + 1);
    } else if (a.bprev0) {
      re = a.bprev0[(b * G + g) * kN + 2 * ri];
      im = a.bprev0[(b * G + g) * kN + 2 * ri + 1];
    }
    float sn, cs;
    __sincosf(phi, &sn, &cs);
    buf[2 * ri] = cs * re - sn * im;
    buf[2 * ri + 1] = sn * re + cs * im;
  };

  float hrow[kPS];  // this thread's row of the state slice
  float phi = 0.f;  // rotation threads: the running angle of pair ri (phi_{t-1} before token t)

  // one forward token: phi_{t-1} -> phi_t, h_{t-1} -> h_t; buffers of t in slot t % 3
  auto fwd_token = [&](int64_t t) {
    const int64_t th = (b * L + t) * H + h;
    const int cur = (int)((t + 3) % 3), prv = (int)((t + 2) % 3);
    if (rot) {
      phi = wrap_angle(phi + (a.theta ? a.theta[th * kNH + ri] : 0.f));
      rot_B(t, phi, Bb[cur]);
    }
    load_x(t, xs[cur]);
    const float at = expf(a.logdecay[th]);
    const float be = a.beta ? a.beta[th] : 0.f, ga = a.gamma[th];
    __syncthreads();
    const float bn = ga * Bb[cur][n], bpn = be * Bb[prv][n];
#pragma unroll
    for (int p = 0; p < kPS; ++p) hrow[p] = fmaf(at, hrow[p], fmaf(bpn, xs[prv][p], bn * xs[cur][p]));
  };
  // the token before t0 into slot (t0 - 1) % 3: Bbar_{t0-1} by phi, x_{t0-1}
  auto prime = [&](int64_t t0) {
    const int slot = (int)((t0 + 2) % 3);
    if (rot) rot_B(t0 - 1, phi, Bb[slot]);
    load_x(t0 - 1, xs[slot]);
  };

  // ---- pass 1: forward with a checkpoint (h_{t0-1}, phi_{t0-1}) every kK tokens ----
  if (rot) phi = wrap_angle(a.angle0 ? a.angle0[bh * kNH + ri] : 0.f);
#pragma unroll
  for (int p = 0; p < kPS; ++p) hrow[p] = a.h0 ? a.h0[(bh * kN + n) * P + p0 + p] : 0.f;
  prime(0);
  for (int64_t t = 0; t < L; ++t) {
    if (t % kK == 0) {
      float* c = chk + (t / kK) * (kN * kPS + kNH);
#pragma unroll
      for (int p = 0; p < kPS; p += 4)
        *reinterpret_cast<float4*>(c + n * kPS + p) =
            make_float4(hrow[p], hrow[p + 1], hrow[p + 2], hrow[p + 3]);
      if (rot) c[kN * kPS + ri] = phi;
    }
    fwd_token(t);
  }

  // ---- pass 2: blocks in reverse ----
  float gS[kPS];     // dL/dh of this row, before the pending decay apend
#pragma unroll
  for (int p = 0; p < kPS; ++p) gS[p] = a.dhT ? a.dhT[(bh * kN + n) * P + p0 + p] : 0.f;
  float apend = 1.f;
  float dxc = 0.f;                      // lanes < kPS of warp 0: gradient of x_{t-1} carried back
  float dbc0 = 0.f, dbc1 = 0.f, dphc = 0.f, rth = 0.f;  // rotation threads: carries of pair ri
  float dDacc = 0.f;                    // thread 0: running dy . x

  for (int64_t k = nblk - 1; k >= 0; --k) {
    const int64_t t0 = k * kK, t1 = (t0 + kK < L) ? t0 + kK : L;
    const float* c = chk + k * (kN * kPS + kNH);
    __syncthreads();  // the previous block's sweep is done with the shared buffers
#pragma unroll
    for (int p = 0; p < kPS; p += 4) {
      const float4 v = *reinterpret_cast<const float4*>(c + n * kPS + p);
      hrow[p] = v.x; hrow[p + 1] = v.y; hrow[p + 2] = v.z; hrow[p + 3] = v.w;
      *reinterpret_cast<float4*>(blk + n * kPS + p) = v;
    }
    if (rot) {
      phi = c[kN * kPS + ri];
      phiB[ri] = phi;
    }
    prime(t0);
    for (int64_t t = t0; t < t1; ++t) {
      fwd_token(t);
      const int64_t j = t - t0 + 1;
#pragma unroll
      for (int p = 0; p < kPS; p += 4)
        *reinterpret_cast<float4*>(blk + (j * kN + n) * kPS + p) =
            make_float4(hrow[p], hrow[p + 1], hrow[p + 2], hrow[p + 3]);
      if (rot) phiB[j * kNH + ri] = phi;
    }
    __syncthreads();  // phiB complete; the recompute's own global writes are this thread's rows

    for (int64_t t = t1 - 1; t >= t0; --t) {
      const int64_t j = t - t0 + 1;
      const int64_t th = (b * L + t) * H + h, tg = (b * L + t) * G + g;
      // this row's h_t and h_{t-1}, in flight while the rotations run
      float St[kPS], Sp[kPS];
#pragma unroll
      for (int p = 0; p < kPS; p += 4) {
        const float4 u = *reinterpret_cast<const float4*>(blk + (j * kN + n) * kPS + p);
        const float4 v = *reinterpret_cast<const float4*>(blk + ((j - 1) * kN + n) * kPS + p);
        St[p] = u.x; St[p + 1] = u.y; St[p + 2] = u.z; St[p + 3] = u.w;
        Sp[p] = v.x; Sp[p + 1] = v.y; Sp[p + 2] = v.z; Sp[p + 3] = v.w;
      }
      // phase A: rotated B_t, C_t (by phi_t) and B_{t-1} (by phi_{t-1}); x, x_prev, dy slices
      float cs = 1.f, sn = 0.f, csp = 1.f, snp = 0.f;
      if (rot) {
        const float ph = phiB[j * kNH + ri], php = phiB[(j - 1) * kNH + ri];
        __sincosf(ph, &sn, &cs);
        __sincosf(php, &snp, &csp);
        const int64_t o = tg * kN;
        const float br = ld(Bg, o + 2 * ri), bi = ld(Bg, o + 2 * ri + 1);
        const float cr = ld(Cg, o + 2 * ri), ci = ld(Cg, o + 2 * ri + 1);
        Bb[0][2 * ri] = cs * br - sn * bi;
        Bb[0][2 * ri + 1] = sn * br + cs * bi;
        Cb[2 * ri] = cs * cr - sn * ci;
        Cb[2 * ri + 1] = sn * cr + cs * ci;
        float pr = 0.f, pi = 0.f;
        if (t > 0) {
          pr = ld(Bg, o - G * kN + 2 * ri);
          pi = ld(Bg, o - G * kN + 2 * ri + 1);
        } else if (a.bprev0) {
          pr = a.bprev0[(b * G + g) * kN + 2 * ri];
          pi = a.bprev0[(b * G + g) * kN + 2 * ri + 1];
        }
        Bpb[2 * ri] = csp * pr - snp * pi;
        Bpb[2 * ri + 1] = snp * pr + csp * pi;
      } else if (tid < kPS) {
        xv[tid] = ld(X, th * P + p0 + tid);
        dyv[tid] = ld(dY, th * P + p0 + tid);
      } else if (tid < 2 * kPS) {
        const int q = tid - kPS;
        xpv[q] = t > 0 ? ld(X, (th - H) * P + p0 + q) : (a.xprev0 ? a.xprev0[bh * P + p0 + q] : 0.f);
      }
      const float at = expf(a.logdecay[th]);
      const float be = a.beta ? a.beta[th] : 0.f, ga = a.gamma[th];
      __syncthreads();  // (1)

      // phase B: this row's element pass, and its shares of <g, h_{t-1}>,
      // dgamma = Bbar_t . (g x_t) and dbeta = Bbar_{t-1} . (g x_{t-1})
      {
        const float cn = Cb[n];
        float rc = 0.f, rx = 0.f, rxp = 0.f, da = 0.f;
#pragma unroll
        for (int p = 0; p < kPS; p += 4) {
          const float4 dy4 = *reinterpret_cast<const float4*>(dyv + p);
          const float4 x4 = *reinterpret_cast<const float4*>(xv + p);
          const float4 xp4 = *reinterpret_cast<const float4*>(xpv + p);
          const float dy[4] = {dy4.x, dy4.y, dy4.z, dy4.w};
          const float xx[4] = {x4.x, x4.y, x4.z, x4.w};
          const float xp[4] = {xp4.x, xp4.y, xp4.z, xp4.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float gv = fmaf(apend, gS[p + q], cn * dy[q]);
            rc = fmaf(St[p + q], dy[q], rc);
            da = fmaf(gv, Sp[p + q], da);
            rx = fmaf(gv, xx[q], rx);
            rxp = fmaf(gv, xp[q], rxp);
            gS[p + q] = gv;
            gvS[n * kPad + p + q] = gv;
          }
        }
        rcv[n] = rc;
        rxv[n] = rx;
        rxpv[n] = rxp;
        float sg = Bb[0][n] * rx, sb = Bpb[n] * rxp;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          da += __shfl_xor_sync(0xffffffffu, da, o);
          sg += __shfl_xor_sync(0xffffffffu, sg, o);
          sb += __shfl_xor_sync(0xffffffffu, sb, o);
        }
        if (lane == 0) {
          red[0][warp] = da;
          red[1][warp] = sg;
          red[2][warp] = sb;
        }
      }
      __syncthreads();  // (2)

      // phase C: column sums g^T Bbar_t and g^T Bbar_{t-1} over rows, in four parts
      {
        const int p = tid & (kPS - 1), which = (tid >> 4) & 1, q = tid >> 5;
        const float* v = which ? Bpb : Bb[0];
        float acc0 = 0.f, acc1 = 0.f;
#pragma unroll 8
        for (int r = 32 * q; r < 32 * q + 32; r += 2) {
          acc0 = fmaf(gvS[r * kPad + p], v[r], acc0);
          acc1 = fmaf(gvS[(r + 1) * kPad + p], v[r + 1], acc1);
        }
        colp[q][which][p] = acc0 + acc1;
      }
      __syncthreads();  // (3)

      // phase D: dX, the scalar partials, and the rotation adjoints
      if (warp == 0) {
        // lanes < kPS: dX of their column; lanes 0..2: the token's scalar partials
        float sd = 0.f;
        if (lane < kPS) {
          const float pb = colp[0][0][lane] + colp[1][0][lane] + colp[2][0][lane] + colp[3][0][lane];
          const float pbp =
              colp[0][1][lane] + colp[1][1][lane] + colp[2][1][lane] + colp[3][1][lane];
          a.dX[th * P + p0 + lane] = dxc + Dh * dyv[lane] + ga * pb;
          dxc = be * pbp;
          sd = dyv[lane] * xv[lane];
        }
        if (lane < 3) {
          const float v = red[lane][0] + red[lane][1] + red[lane][2] + red[lane][3];
          dScal[th * 3 + lane] = lane == 0 ? at * v : v;
        }
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) sd += __shfl_xor_sync(0xffffffffu, sd, o);
        if (lane == 0) dDacc += sd;
      } else if (rot) {
        const float d0 = ga * rxv[2 * ri], d1 = ga * rxv[2 * ri + 1];
        const float e0 = rcv[2 * ri], e1 = rcv[2 * ri + 1];
        dBp[th * kN + 2 * ri] = cs * d0 + sn * d1 + dbc0;
        dBp[th * kN + 2 * ri + 1] = -sn * d0 + cs * d1 + dbc1;
        dCp[th * kN + 2 * ri] = cs * e0 + sn * e1;
        dCp[th * kN + 2 * ri + 1] = -sn * e0 + cs * e1;
        const float dph = -d0 * Bb[0][2 * ri + 1] + d1 * Bb[0][2 * ri] - e0 * Cb[2 * ri + 1] +
                          e1 * Cb[2 * ri] + dphc;
        rth += dph;
        dThp[th * kNH + ri] = rth;
        const float f0 = be * rxpv[2 * ri], f1 = be * rxpv[2 * ri + 1];
        dbc0 = csp * f0 + snp * f1;
        dbc1 = -snp * f0 + csp * f1;
        dphc = -f0 * Bpb[2 * ri + 1] + f1 * Bpb[2 * ri];
      }
      apend = at;
      __syncthreads();  // (4)
    }
  }

  // ---- gradients of the initial state and the cache inputs ----
  if (a.dh0) {
#pragma unroll
    for (int p = 0; p < kPS; ++p) a.dh0[(bh * kN + n) * P + p0 + p] = apend * gS[p];
  }
  if (a.dxprev0 && tid < kPS) a.dxprev0[bh * P + p0 + tid] = dxc;
  if (rot) {
    dbpp[bh * kN + 2 * ri] = dbc0;
    dbpp[bh * kN + 2 * ri + 1] = dbc1;
    dAngp[bh * kNH + ri] = rth + dphc;
  }
  if (tid == 0) dDp[bh] = dDacc;
}

// Sums of the slice partials (and of the heads of a group, and of the batch for
// dD), each in a fixed order.
__global__ void bwd_split_reduce_kernel(BwdArgs a, SplitWs ws) {
  const int64_t H = a.H, G = a.G, hpg = H / G, S = a.P / kPS;
  const int64_t th = a.b * a.L * H, tg = a.b * a.L * G, bh = a.b * H, bg = a.b * G;
  const char* wsb = static_cast<const char*>(a.workspace);
  const float* dBp = reinterpret_cast<const float*>(wsb + ws.dBp);
  const float* dCp = reinterpret_cast<const float*>(wsb + ws.dCp);
  const float* dThp = reinterpret_cast<const float*>(wsb + ws.dThp);
  const float* dScal = reinterpret_cast<const float*>(wsb + ws.dScal);
  const float* dbpp = reinterpret_cast<const float*>(wsb + ws.dbpp);
  const float* dAngp = reinterpret_cast<const float*>(wsb + ws.dAngp);
  const float* dDp = reinterpret_cast<const float*>(wsb + ws.dDp);
  const int64_t nBC = tg * kN, nTh = th * kNH, nSc = th, nbp = bg * kN, nAng = bh * kNH;
  const int64_t total = nBC + nTh + nSc + nbp + nAng + H;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
    int64_t r = i;
    if (r < nBC) {  // dB, dC: (b, L, G, N)
      const int64_t nn = r % kN, row = r / kN, gg = row % G, bt = row / G;
      float sbv = 0.f, scv = 0.f;
      for (int64_t q = 0; q < hpg; ++q) {
        const int64_t src = (bt * H + gg * hpg + q) * kN + nn;
        for (int64_t sl = 0; sl < S; ++sl) {
          sbv += dBp[sl * th * kN + src];
          scv += dCp[sl * th * kN + src];
        }
      }
      a.dB[r] = sbv;
      a.dC[r] = scv;
      continue;
    }
    r -= nBC;
    if (r < nTh) {  // dtheta: (b, L, H, N/2)
      float v = 0.f;
      for (int64_t sl = 0; sl < S; ++sl) v += dThp[sl * nTh + r];
      if (a.dtheta) a.dtheta[r] = v;
      continue;
    }
    r -= nTh;
    if (r < nSc) {  // dlogdecay, dgamma, dbeta: (b, L, H)
      float v0 = 0.f, v1 = 0.f, v2 = 0.f;
      for (int64_t sl = 0; sl < S; ++sl) {
        v0 += dScal[(sl * th + r) * 3 + 0];
        v1 += dScal[(sl * th + r) * 3 + 1];
        v2 += dScal[(sl * th + r) * 3 + 2];
      }
      a.dlogdecay[r] = v0;
      a.dgamma[r] = v1;
      if (a.dbeta) a.dbeta[r] = v2;
      continue;
    }
    r -= nSc;
    if (r < nbp) {  // dbprev0: (b, G, N)
      const int64_t nn = r % kN, row = r / kN, gg = row % G, bb = row / G;
      float v = 0.f;
      for (int64_t q = 0; q < hpg; ++q)
        for (int64_t sl = 0; sl < S; ++sl) v += dbpp[(sl * bh + bb * H + gg * hpg + q) * kN + nn];
      if (a.dbprev0) a.dbprev0[r] = v;
      continue;
    }
    r -= nbp;
    if (r < nAng) {  // dangle0: (b, H, N/2)
      float v = 0.f;
      for (int64_t sl = 0; sl < S; ++sl) v += dAngp[sl * nAng + r];
      if (a.dangle0) a.dangle0[r] = v;
      continue;
    }
    r -= nAng;
    {  // dD: (H)
      float v = 0.f;
      for (int64_t bb = 0; bb < a.b; ++bb)
        for (int64_t sl = 0; sl < S; ++sl) v += dDp[sl * bh + bb * H + r];
      if (a.dD) a.dD[r] = v;
    }
  }
}

}  // namespace

bool bwd_split_supported(int64_t N, int64_t P) { return N == kN && P % kPS == 0 && P >= kPS; }

size_t bwd_split_workspace_bytes(int64_t b, int64_t L, int64_t H, int64_t P) {
  return split_ws_layout(b, L, H, P).total;
}

cudaError_t launch_bwd_split(const BwdArgs& a, cudaStream_t s) {
  if (a.b * a.H == 0) return cudaSuccess;
  const SplitWs ws = split_ws_layout(a.b, a.L, a.H, a.P);
  const unsigned grid = (unsigned)(a.b * a.H * (a.P / kPS));
  if (a.bf16)
    bwd_split_kernel<__nv_bfloat16><<<grid, kT, 0, s>>>(a, ws);
  else
    bwd_split_kernel<float><<<grid, kT, 0, s>>>(a, ws);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t total = a.b * a.L * a.G * kN + a.b * a.L * a.H * (kNH + 1) + a.b * a.G * kN +
                        a.b * a.H * kNH + a.H;
  const unsigned rg = (unsigned)((total + 255) / 256 < 148 * 32 ? (total + 255) / 256 : 148 * 32);
  bwd_split_reduce_kernel<<<rg > 0 ? rg : 1, 256, 0, s>>>(a, ws);
  return cudaGetLastError();
}

}  // namespace m3ssd
