// Chunked bf16 forward of the Mamba-3 SISO scan (N = 128, P = 64).
//
// One CTA owns one (b, h) sequence and walks its chunks in order, keeping the
// fp32 state h on chip for the whole sequence (no chunk state goes to HBM).
//
// Chunk layout.  Chunk c has Q = 64 source rows: row 0 is the token just
// before the chunk (t0 - 1, the carry-in of the trapezoid's beta term) and rows
// 1..63 are the chunk's own tokens t0 .. t0+62 (t0 = 63 c).  With the running
// angle phi and the chunk-local sums (row 0 has cs_0 = 0, psi_0 = 0)
//     cs_r = sum_{k=1..r} logdecay_k,   psi_r = sum_{k=1..r} theta_k,
// the rotated vectors are Bbar_r = R(Phi_c + psi_r) B_r, Cbar_r likewise, where
// Phi_c = phi_{t0-1} is carried from chunk to chunk, and the recurrence
// ("TorchMamba" README, "Math notes", M3 SISO: exponential-trapezoidal update
// h_t = alpha_t h_{t-1} + beta_t Bbar_{t-1} x_{t-1}^T + gamma_t Bbar_t x_t^T)
// unrolled over the chunk reads, for output rows r = 1..63,
//     y_r   = exp(cs_r) Cbar_r^T h + sum_{u<=r} W(r,u) (Cbar_r^T Bbar_u) x_u + D x_r
//     h_end = exp(cs_63) h + sum_u W(63,u) Bbar_u x_u^T
//     W(r,r) = gamma_r,   W(r,u<r) = exp(cs_r - cs_{u+1}) (gamma_u alpha_{u+1} + beta_{u+1}),
// with gamma_0 := 0 (row 0's own gamma term belongs to the previous chunk), so
// the column u = 0 carries exactly the beta boundary term.  The gamma and beta
// terms form one mask ("TorchMamba" README: "the parallel mask is L = 1SS @
// band") applied to the Gram matrix in a single pass.
//
// Tensor-core work per chunk (mma.sync m16n8k16, bf16 in, fp32 accumulate):
//   G   = Cbar Bbar^T                 lower-triangular 16x8 tiles only
//   Y   = diag(exp cs) Cbar h  +  (W o G) X
//   h   = exp(cs_63) h + (W_end o Bbar)^T X, with W_end o Bbar split into a
//         bf16 high part and a bf16 residual so the state update carries one
//         rounding of ~2^-17 instead of two of 2^-9 (X itself is exact bf16).
// Decay/angle cumsums, sincos, rotations, masks and epilogues run on the SIMT
// pipes.  Shared tiles use a 16-byte XOR swizzle so ldmatrix is conflict-free
// without padding, which keeps two CTAs resident per SM.
#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"

namespace m3ssd {
namespace {

constexpr int Q = 64;       // source rows per chunk (1 carry-in + 63 tokens)
constexpr int QT = Q - 1;   // tokens per chunk
constexpr int NS = 128;     // state size N
constexpr int PD = 64;      // head dim P
constexpr int NH = NS / 2;  // rotation pairs
constexpr int kThreads = 256;
constexpr float kLog2e = 1.4426950408889634f;

typedef __nv_bfloat16 bf16;

// 16-byte-chunk XOR swizzle of a row-major bf16 tile with RL elements a row.
template <int RL>
__device__ __forceinline__ int swz(int r, int c) {
  return r * RL + ((((c >> 3) ^ (r & 7))) << 3) + (c & 7);
}

struct Smem {
  union {
    float theta[Q][NH];  // raw theta of the chunk (phase R1 only)
    bf16 bw_hi[Q * NS];  // high part of W_end o Bbar (phase R2 .. S)
  } u;
  bf16 bw_lo[Q * NS];    // residual of W_end o Bbar
  bf16 B[Q * NS];        // raw B, then Bbar
  bf16 C[Q * NS];        // raw C, then Cbar
  bf16 X[Q * PD];        // X rows of the chunk (row 0 = carry-in token)
  bf16 M[Q * Q];         // masked Gram W o G
  bf16 Hs[NS * PD];      // bf16 copy of h for the state-to-output product
  float segtot[4][NH];
  float cs2[Q], ecs[Q], cvec[Q], wend[Q], gam[Q];
  float ecos[NH], esin[NH], Phi[NH];  // exp(i Phi_c) per pair and Phi_c itself
  float necos[NH], nesin[NH], nPhi[NH];  // the same for the next chunk
  float scal[4];
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(dst)), "l"(src),
               "r"(valid ? 16 : 0));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;\n" ::); }

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}
// D += A * B, m16n8k16, bf16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}

// Lower-triangular 16x8 tile u (0..19) of the 64x64 Gram: block row bi, column tile nj.
__device__ __forceinline__ void gram_unit(int u, int& bi, int& nj) {
  bi = (u < 2) ? 0 : (u < 6) ? 1 : (u < 12) ? 2 : 3;
  nj = u - bi * (bi + 1);
}

template <bool ROT>
__global__ void __launch_bounds__(kThreads, 2) fwd_chunk_kernel(FwdArgs a) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t H = a.H, L = a.L, G = a.G;
  const int64_t bh = blockIdx.x;
  const int64_t b = bh / H, h = bh % H, g = h / (H / G);
  const int nC = (int)((L + QT - 1) / QT);
  const bf16* Xg = static_cast<const bf16*>(a.X);
  const bf16* Bg = static_cast<const bf16*>(a.B);
  const bf16* Cg = static_cast<const bf16*>(a.C);
  bf16* Yg = static_cast<bf16*>(a.Y);
  const float Dh = a.D ? a.D[h] : 0.f;

  // Row r of chunk c holds token c*QT - 1 + r; rows outside [0, L) are zero-filled.
  auto row_token = [&](int c, int r) -> int64_t { return (int64_t)c * QT - 1 + r; };
  auto load_theta = [&](int c) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int idx = tid + k * kThreads;
      const int row = idx >> 4, col = (idx & 15) * 4;
      const int64_t t = row_token(c, row);
      const bool ok = a.theta && t >= 0 && t < L;
      const float* src = ok ? a.theta + ((b * L + t) * H + h) * NH + col : a.logdecay;
      cp_async16(&sm.u.theta[row][col], src, ok);
    }
  };
  auto load_b = [&](int c, const bf16* base, bf16* dst) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int idx = tid + k * kThreads;
      const int row = idx >> 4, col = (idx & 15) * 8;
      const int64_t t = row_token(c, row);
      const bool ok = t >= 0 && t < L;
      const bf16* src = ok ? base + ((b * L + t) * G + g) * NS + col : base;
      if (t >= 0) cp_async16(&dst[swz<NS>(row, col)], src, ok);
    }
  };
  auto load_x = [&](int c) {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int idx = tid + k * kThreads;
      const int row = idx >> 3, col = (idx & 7) * 8;
      const int64_t t = row_token(c, row);
      const bool ok = t >= 0 && t < L;
      const bf16* src = ok ? Xg + ((b * L + t) * H + h) * PD + col : Xg;
      if (t >= 0) cp_async16(&sm.X[swz<PD>(row, col)], src, ok);
    }
  };
  // warp 0 keeps logdecay / beta / gamma of rows lane and lane + 32 in registers
  float pld[2], pbe[2], pga[2];
  auto load_params = [&](int c) {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int r = lane + 32 * k;
      const int64_t t = row_token(c, r);
      const bool ok = r > 0 && t < L;  // row 0 (carry-in) has a = gamma = beta = 0 here
      const int64_t idx = (b * L + (ok ? t : 0)) * H + h;
      pld[k] = ok ? a.logdecay[idx] : 0.f;
      pga[k] = ok ? a.gamma[idx] : 0.f;
      pbe[k] = (ok && a.beta) ? a.beta[idx] : 0.f;
    }
  };

  // ---- prologue -------------------------------------------------------------
  if (ROT) load_theta(0);
  load_b(0, Bg, sm.B);
  load_b(0, Cg, sm.C);
  load_x(0);
  cp_async_commit();
  if (warp == 0) load_params(0);
  // row 0 of chunk 0 is the cache's previous token (zero when absent)
  if (tid < NS) {
    sm.B[swz<NS>(0, tid)] = __float2bfloat16_rn(a.bprev0 ? a.bprev0[(b * G + g) * NS + tid] : 0.f);
    sm.C[swz<NS>(0, tid)] = __float2bfloat16_rn(0.f);
  }
  if (tid < PD) sm.X[swz<PD>(0, tid)] = __float2bfloat16_rn(a.xprev0 ? a.xprev0[bh * PD + tid] : 0.f);
  if (ROT && tid < NH) {
    const float ph0 = a.angle0 ? a.angle0[bh * NH + tid] : 0.f;
    sm.Phi[tid] = ph0;
    float s, c;
    sincosf(ph0, &s, &c);
    sm.ecos[tid] = c;
    sm.esin[tid] = s;
  }

  // state fragment: rows rb + mi*16 + lane/4 (+8), cols ph*32 + j*8 + 2*(lane%4) (+1)
  const int rb = 32 * (warp & 3), ph = warp >> 2;
  float hs[2][4][4];
#pragma unroll
  for (int mi = 0; mi < 2; ++mi)
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int n = rb + mi * 16 + (lane >> 2) + 8 * hf;
        const int p = ph * 32 + j * 8 + 2 * (lane & 3);
        float2 v = make_float2(0.f, 0.f);
        if (a.h0) v = *reinterpret_cast<const float2*>(&a.h0[(bh * NS + n) * PD + p]);
        hs[mi][j][2 * hf] = v.x;
        hs[mi][j][2 * hf + 1] = v.y;
      }
  auto store_state_bf16 = [&]() {
#pragma unroll
    for (int mi = 0; mi < 2; ++mi)
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int n = rb + mi * 16 + (lane >> 2) + 8 * hf;
          const int p = ph * 32 + j * 8 + 2 * (lane & 3);
          *reinterpret_cast<uint32_t*>(&sm.Hs[swz<PD>(n, p)]) =
              pack_bf16(hs[mi][j][2 * hf], hs[mi][j][2 * hf + 1]);
        }
  };
  store_state_bf16();

  // ---- chunk walk -------------------------------------------------------------
  for (int c = 0; c < nC; ++c) {
    const int64_t tbase = (int64_t)c * QT - 1;  // token of row 0
    cp_async_wait_all();
    __syncthreads();  // S1: theta, B, C, X of this chunk are in shared memory

    // -- phase R1: decay cumsum and chunk parameters (warp 0), angle cumsum -------
    if (warp == 0) {
      float s0 = pld[0], s1 = pld[1];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float u0 = __shfl_up_sync(0xffffffffu, s0, o);
        const float u1 = __shfl_up_sync(0xffffffffu, s1, o);
        if (lane >= o) { s0 += u0; s1 += u1; }
      }
      s1 += __shfl_sync(0xffffffffu, s0, 31);
      const float cs[2] = {s0, s1};
      const float cs_end = __shfl_sync(0xffffffffu, s1, 31);
      const float ld_dn0 = __shfl_down_sync(0xffffffffu, pld[0], 1);
      const float ld_dn1 = __shfl_down_sync(0xffffffffu, pld[1], 1);
      const float be_dn0 = __shfl_down_sync(0xffffffffu, pbe[0], 1);
      const float be_dn1 = __shfl_down_sync(0xffffffffu, pbe[1], 1);
      const float cs_dn0 = __shfl_down_sync(0xffffffffu, s0, 1);
      const float cs_dn1 = __shfl_down_sync(0xffffffffu, s1, 1);
      const float ld_32 = __shfl_sync(0xffffffffu, pld[1], 0);
      const float be_32 = __shfl_sync(0xffffffffu, pbe[1], 0);
      const float cs_32 = __shfl_sync(0xffffffffu, s1, 0);
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int r = lane + 32 * k;
        const float ld_next = k == 0 ? (lane < 31 ? ld_dn0 : ld_32) : ld_dn1;
        const float be_next = k == 0 ? (lane < 31 ? be_dn0 : be_32) : be_dn1;
        const float cs_next = k == 0 ? (lane < 31 ? cs_dn0 : cs_32) : cs_dn1;
        sm.cs2[r] = cs[k] * kLog2e;
        sm.ecs[r] = expf(cs[k]);
        sm.gam[r] = pga[k];
        if (r < Q - 1) {
          const float cv = pga[k] * expf(ld_next) + be_next;
          sm.cvec[r] = cv;
          sm.wend[r] = expf(cs_end - cs_next) * cv;
        } else {
          sm.cvec[r] = pga[k];
          sm.wend[r] = pga[k];
        }
      }
      if (lane == 0) sm.scal[0] = expf(cs_end);
      if (c + 1 < nC) load_params(c + 1);
    }
    const int pi = tid & 63, seg = tid >> 6;
    float psi[16];
    if (ROT) {
      float run = 0.f;
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        if (seg > 0 || k > 0) run += sm.u.theta[seg * 16 + k][pi];  // psi_0 = 0
        psi[k] = run;
      }
      sm.segtot[seg][pi] = run;
    }
    __syncthreads();  // S2: parameters ready; theta no longer read

    // -- phase R2: rotation into the absolute frame, W_end o Bbar hi/lo ----------
    {
      float off = 0.f, ec = 1.f, es = 0.f;
      if (ROT) {
        for (int s2 = 0; s2 < seg; ++s2) off += sm.segtot[s2][pi];
        ec = sm.ecos[pi];
        es = sm.esin[pi];
      }
#pragma unroll 4
      for (int k = 0; k < 16; ++k) {
        const int r = seg * 16 + k;
        uint32_t* pb = reinterpret_cast<uint32_t*>(&sm.B[swz<NS>(r, 2 * pi)]);
        uint32_t* pc = reinterpret_cast<uint32_t*>(&sm.C[swz<NS>(r, 2 * pi)]);
        float2 bv = unpack_bf16(*pb);
        float2 cv = unpack_bf16(*pc);
        if (ROT) {
          float s, co;
          fast_sincos(psi[k] + off, &s, &co);
          // exp(i (Phi_c + psi)) = exp(i Phi_c) exp(i psi)
          const float cr = ec * co - es * s, sr = es * co + ec * s;
          bv = rot2(cr, sr, bv.x, bv.y);
          cv = rot2(cr, sr, cv.x, cv.y);
          *pb = pack_bf16(bv.x, bv.y);
          *pc = pack_bf16(cv.x, cv.y);
        }
        const float we = sm.wend[r];
        const float w0 = we * bv.x, w1 = we * bv.y;
        const uint32_t hi = pack_bf16(w0, w1);
        const float2 hv = unpack_bf16(hi);
        *reinterpret_cast<uint32_t*>(&sm.u.bw_hi[swz<NS>(r, 2 * pi)]) = hi;
        *reinterpret_cast<uint32_t*>(&sm.bw_lo[swz<NS>(r, 2 * pi)]) = pack_bf16(w0 - hv.x, w1 - hv.y);
      }
      if (ROT && seg == 3) {
        const float pnext = wrap_angle(sm.Phi[pi] + psi[15] + off);
        float s, co;
        sincosf(pnext, &s, &co);
        sm.nPhi[pi] = pnext;
        sm.necos[pi] = co;
        sm.nesin[pi] = s;
      }
    }
    __syncthreads();  // S3: Bbar, Cbar, W_end o Bbar ready
    if (ROT && tid < NH) {
      sm.Phi[tid] = sm.nPhi[tid];
      sm.ecos[tid] = sm.necos[tid];
      sm.esin[tid] = sm.nesin[tid];
    }

    // -- phase G: masked Gram -> M ---------------------------------------------
    for (int u = warp; u < 20; u += 8) {
      int bi, nj;
      gram_unit(u, bi, nj);
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int kk = 0; kk < 8; kk += 2) {
        uint32_t bfr[4];
        ldsm_x4(bfr, &sm.B[swz<NS>(nj * 8 + (lane & 7), kk * 16 + 8 * (lane >> 3))]);
#pragma unroll
        for (int k2 = 0; k2 < 2; ++k2) {
          uint32_t afr[4];
          ldsm_x4(afr, &sm.C[swz<NS>(bi * 16 + (lane & 7) + 8 * ((lane >> 3) & 1),
                                     (kk + k2) * 16 + 8 * (lane >> 4))]);
          mma16816(acc, afr, bfr[2 * k2], bfr[2 * k2 + 1]);
        }
      }
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int t = bi * 16 + (lane >> 2) + 8 * hf;
        const int s0 = nj * 8 + 2 * (lane & 3);
        float w[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int s = s0 + j;
          w[j] = (s > t) ? 0.f
                 : (s == t) ? sm.gam[t]
                            : exp2f(sm.cs2[t] - sm.cs2[s + 1]) * sm.cvec[s];
        }
        *reinterpret_cast<uint32_t*>(&sm.M[swz<Q>(t, s0)]) =
            pack_bf16(acc[2 * hf] * w[0], acc[2 * hf + 1] * w[1]);
      }
    }
    __syncthreads();  // S4: M ready; Bbar (sm.B) is free
    if (c + 1 < nC) {
      load_b(c + 1, Bg, sm.B);
      cp_async_commit();
    }

    // -- phase Y: outputs, 16 rows x 32 columns per warp ------------------------
    {
      const int mt = warp & 3;
      float acc[4][4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[j][e] = 0.f;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        uint32_t afr[4];
        ldsm_x4(afr, &sm.C[swz<NS>(mt * 16 + (lane & 7) + 8 * ((lane >> 3) & 1),
                                   kk * 16 + 8 * (lane >> 4))]);
#pragma unroll
        for (int np = 0; np < 2; ++np) {
          uint32_t bfr[4];
          ldsm_x4_t(bfr, &sm.Hs[swz<PD>(kk * 16 + (lane & 7) + 8 * ((lane >> 3) & 1),
                                        ph * 32 + np * 16 + 8 * (lane >> 4))]);
          mma16816(acc[2 * np], afr, bfr[0], bfr[1]);
          mma16816(acc[2 * np + 1], afr, bfr[2], bfr[3]);
        }
      }
      const float e_lo = sm.ecs[mt * 16 + (lane >> 2)];
      const float e_hi = sm.ecs[mt * 16 + (lane >> 2) + 8];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        acc[j][0] *= e_lo; acc[j][1] *= e_lo;
        acc[j][2] *= e_hi; acc[j][3] *= e_hi;
      }
      for (int kk = 0; kk <= mt; ++kk) {
        uint32_t afr[4];
        ldsm_x4(afr, &sm.M[swz<Q>(mt * 16 + (lane & 7) + 8 * ((lane >> 3) & 1),
                                  kk * 16 + 8 * (lane >> 4))]);
#pragma unroll
        for (int np = 0; np < 2; ++np) {
          uint32_t bfr[4];
          ldsm_x4_t(bfr, &sm.X[swz<PD>(kk * 16 + (lane & 7) + 8 * ((lane >> 3) & 1),
                                       ph * 32 + np * 16 + 8 * (lane >> 4))]);
          mma16816(acc[2 * np], afr, bfr[0], bfr[1]);
          mma16816(acc[2 * np + 1], afr, bfr[2], bfr[3]);
        }
      }
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int r = mt * 16 + (lane >> 2) + 8 * hf;
        const int64_t t = tbase + r;
        if (r > 0 && t < L) {
          bf16* yrow = Yg + ((b * L + t) * H + h) * PD;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int p = ph * 32 + j * 8 + 2 * (lane & 3);
            const float2 xv = unpack_bf16(*reinterpret_cast<const uint32_t*>(&sm.X[swz<PD>(r, p)]));
            *reinterpret_cast<uint32_t*>(yrow + p) =
                pack_bf16(acc[j][2 * hf] + Dh * xv.x, acc[j][2 * hf + 1] + Dh * xv.y);
          }
        }
      }
    }
    __syncthreads();  // S5: readers of Hs and Cbar are done
    if (c + 1 < nC) {
      load_b(c + 1, Cg, sm.C);
      cp_async_commit();
    }

    // -- phase S: h = exp(cs_end) h + (W_end o Bbar)^T X ---------------------------
    {
      const float eE = sm.scal[0];
#pragma unroll
      for (int mi = 0; mi < 2; ++mi)
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int e = 0; e < 4; ++e) hs[mi][j][e] *= eE;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        uint32_t bx[2][4];
#pragma unroll
        for (int np = 0; np < 2; ++np)
          ldsm_x4_t(bx[np], &sm.X[swz<PD>(kk * 16 + (lane & 7) + 8 * ((lane >> 3) & 1),
                                          ph * 32 + np * 16 + 8 * (lane >> 4))]);
#pragma unroll
        for (int mi = 0; mi < 2; ++mi) {
          const int arow = kk * 16 + (lane & 7) + 8 * (lane >> 4);
          const int acol = rb + mi * 16 + 8 * ((lane >> 3) & 1);
          uint32_t ahi[4], alo[4];
          ldsm_x4_t(ahi, &sm.u.bw_hi[swz<NS>(arow, acol)]);
          ldsm_x4_t(alo, &sm.bw_lo[swz<NS>(arow, acol)]);
#pragma unroll
          for (int np = 0; np < 2; ++np) {
            mma16816(hs[mi][2 * np], ahi, bx[np][0], bx[np][1]);
            mma16816(hs[mi][2 * np + 1], ahi, bx[np][2], bx[np][3]);
            mma16816(hs[mi][2 * np], alo, bx[np][0], bx[np][1]);
            mma16816(hs[mi][2 * np + 1], alo, bx[np][2], bx[np][3]);
          }
        }
      }
      store_state_bf16();
    }
    __syncthreads();  // S6: theta / W_end o Bbar / X buffers are free
    if (c + 1 < nC) {
      if (ROT) load_theta(c + 1);
      load_x(c + 1);
      cp_async_commit();
    }
  }
  cp_async_wait_all();

  // ---- outputs of the last token ----------------------------------------------
  if (a.hT) {
#pragma unroll
    for (int mi = 0; mi < 2; ++mi)
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int n = rb + mi * 16 + (lane >> 2) + 8 * hf;
          const int p = ph * 32 + j * 8 + 2 * (lane & 3);
          *reinterpret_cast<float2*>(&a.hT[(bh * NS + n) * PD + p]) =
              make_float2(hs[mi][j][2 * hf], hs[mi][j][2 * hf + 1]);
        }
  }
  if (a.angleT && tid < NH)
    a.angleT[bh * NH + tid] = ROT ? sm.Phi[tid] : (a.angle0 ? a.angle0[bh * NH + tid] : 0.f);
  if (a.xprevT && tid < PD) a.xprevT[bh * PD + tid] = __bfloat162float(Xg[((b * L + L - 1) * H + h) * PD + tid]);
  if (a.bprevT && h % (H / G) == 0 && tid < NS)
    a.bprevT[(b * G + g) * NS + tid] = __bfloat162float(Bg[((b * L + L - 1) * G + g) * NS + tid]);
}

template <bool ROT>
cudaError_t launch_variant(const FwdArgs& a, cudaStream_t s) {
  const size_t smem = sizeof(Smem);
  cudaError_t e = cudaFuncSetAttribute(fwd_chunk_kernel<ROT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  fwd_chunk_kernel<ROT><<<(unsigned)(a.b * a.H), kThreads, smem, s>>>(a);
  return cudaGetLastError();
}

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

bool fwd_chunk_supported(const FwdArgs& a) {
  return a.bf16 && a.N == NS && a.P == PD && a.L > 0 && (a.chunk == 0 || a.chunk == Q) &&
         al16(a.X) && al16(a.B) && al16(a.C) && al16(a.Y) && al16(a.theta) && al16(a.h0) &&
         al16(a.hT) && al16(a.logdecay);
}

cudaError_t launch_fwd_chunk(const FwdArgs& a, cudaStream_t s) {
  if (a.b * a.H == 0) return cudaSuccess;
  if (a.theta != nullptr || a.angle0 != nullptr) return launch_variant<true>(a, s);
  return launch_variant<false>(a, s);
}

}  // namespace m3ssd
