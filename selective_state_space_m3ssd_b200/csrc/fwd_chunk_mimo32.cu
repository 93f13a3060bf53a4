// Chunked forward of the Mamba-3 MIMO scan for fp32 X, B, C, Y at rank R = 2, 4
// or 8, N = 128, P = 64, on the sm_100a tensor cores with every product on fp16
// high / low operand parts.
//
// The chunk is the bf16 MIMO kernel's (64 rows of (token, rank), 64/R - 1 new
// tokens and the carry-in token, the trapezoid weight of a token pair over an
// R x R block of the mask; "TorchMamba" README, "Math notes", MIMO), and the
// precision is the fp32 SISO kernel's: each operand v is hi = fp16(v) and
// lo = fp16(v - hi), each product hi.hi + hi.lo + lo.hi (about 2^-22 of each term
// in fp16's normal range), the state copy scaled by a power of two.
//
// Shared memory: the fp32 inputs keep the rank axis innermost in HBM.  A 4-D
// tensor map over (N R, group, token, batch) with a box of 32 R values lands
// n-block k (n in [32k, 32k+32), every rank) of all the chunk's tokens in the
// high atom k/2 (k even) or the low atom k/2 (k odd) of the operand tile, so a
// token's 256 R raw bytes of one half of N are exactly the bytes of its R rows
// in that half's high and low atoms; one warp per (token, half) reads them all
// and converts in place (X likewise with p-blocks of 32).  Y (fp32) is staged
// through the masked Gram's 16 KB once Y2 has read it and leaves in 16-byte
// stores.  One CTA per SM (about 170 KB of shared memory).
#include <cuda.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <cstring>

#include "common.cuh"
#include "internal.h"
#include "mimo_chunk.cuh"
#include "tc5.cuh"

namespace m3ssd {

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

__device__ unsigned int g_mimo32_wait_timeouts;

namespace {

using namespace chunk;
using mchunk::MParams;
using mchunk::chunk_params;

constexpr int kCtrlWarp = 8;
constexpr int kThreads = 32 * (kCtrlWarp + 1);
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColG = 0, kColY1 = 64, kColY2 = 128, kColS = 192;
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr uint32_t kIdescG = tc5::idesc_f16(64, 64, false, false);
constexpr uint32_t kIdescY = tc5::idesc_f16(64, 64, false, true);
constexpr uint32_t kIdescS = tc5::idesc_f16(128, 64, true, true);

// 2R floats (8R bytes, 16-byte aligned) of shared memory into registers
template <int R>
__device__ __forceinline__ void lds_f(const uint8_t* p, float (&v)[2 * R]) {
#pragma unroll
  for (int i = 0; i < R / 2; ++i) {
    const float4 w = reinterpret_cast<const float4*>(p)[i];
    v[4 * i] = w.x; v[4 * i + 1] = w.y; v[4 * i + 2] = w.z; v[4 * i + 3] = w.w;
  }
}

struct MSmem32 {
  float ang[32][NH];           // theta of the chunk's token rows, then their absolute angles
  uint8_t wx[2 * kAtom];       // W_end o X: high atom, low atom
  uint8_t B[4 * kAtom];        // raw n-blocks 0..3, then Bbar: high 0, low 0, high 1, low 1
  uint8_t C[4 * kAtom];        // the same for C
  uint8_t X[2][2 * kAtom];     // raw p-blocks 0, 1, then X: high, low (chunks c, c + 1)
  uint8_t M[2 * kAtom];        // masked Gram high, low; after Y2 the chunk's fp32 Y in HBM order
  uint8_t Hs[2 * NS * 128];    // h 2^k: high, low
  float hmax[8];
  MParams prm[2];
  float segtot[4][NH];
  float Phi[NH];
  float nPhi[NH];
  uint64_t mbar[4];
  uint64_t lmbar;
  uint32_t tmem;
  uint32_t err;
};
static_assert(sizeof(MSmem32) + 1024 <= 232448, "one CTA per SM");

struct MMaps32 {
  CUtensorMap theta;  // fp32 (pair, head, token, batch), box 64 x 1 x (64/R) x 1
  CUtensorMap B;      // fp32 (N R, group, token, batch), box 32 R x 1 x (64/R) x 1
  CUtensorMap C;
  CUtensorMap X;      // fp32 (P R, head, token, batch), box 32 R x 1 x (64/R) x 1
};

template <int R, bool ROT>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_chunk_mimo32_kernel(FwdArgs a, const __grid_constant__ MMaps32 tm) {
  static_assert(R == 2 || R == 4 || R == 8, "rank");
  constexpr int TQ = Q / R, QT = TQ - 1;
  constexpr int RB = 128 * R;  // bytes of one token's R rows in one atom
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw_addr = tc5::saddr(smem_raw);
  MSmem32& sm = *reinterpret_cast<MSmem32*>(smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool ctrl = warp == kCtrlWarp;
  const bool ctrl_lead = tid == kCtrlWarp * 32;
  const int64_t H = a.H, L = a.L, G = a.G;
  const int64_t bh = blockIdx.x;
  const int64_t b = bh / H, h = bh % H, g = h / (H / G);
  const int nC = (int)((L + QT - 1) / QT);
  const float* Xg = static_cast<const float*>(a.X);
  const float* Bg = static_cast<const float*>(a.B);
  uint8_t* const Yg8 = static_cast<uint8_t*>(a.Y);
  const float Dh = a.D ? a.D[h] : 0.f;
  const uint32_t aB = tc5::saddr(sm.B), aC = tc5::saddr(sm.C);
  const uint32_t aX0 = tc5::saddr(sm.X[0]);
  const uint32_t aM = tc5::saddr(sm.M), aH = tc5::saddr(sm.Hs);
  const uint32_t aWX = tc5::saddr(sm.wx);
  const uint32_t aT = tc5::saddr(&sm.ang[0][0]);
  const bool has_theta = a.theta != nullptr;
  const uint32_t chunk_bytes =
      (ROT && has_theta ? (uint32_t)(TQ * NH * 4) : 0u) + 8u * kAtom + 2u * kAtom;
  auto tma_theta = [&](int c) {
    tc5::tma_load_4d(aT, &tm.theta, &sm.lmbar, 0, (int)h, c * QT - 1, (int)b);
  };
  auto tma_bc = [&](int c, const CUtensorMap* map, uint32_t base) {
#pragma unroll
    for (int k = 0; k < 4; ++k)
      tc5::tma_load_4d(base + (uint32_t)k * kAtom, map, &sm.lmbar, 32 * R * k, (int)g, c * QT - 1,
                       (int)b);
  };
  auto tma_x = [&](int c) {
    const uint32_t base = aX0 + (uint32_t)(c & 1) * (2 * kAtom);
    tc5::tma_load_4d(base, &tm.X, &sm.lmbar, 0, (int)h, c * QT - 1, (int)b);
    tc5::tma_load_4d(base + kAtom, &tm.X, &sm.lmbar, 32 * R, (int)h, c * QT - 1, (int)b);
  };
  float pld = 0.f, pbe = 0.f, pga = 0.f;
  auto load_params = [&](int c) {
    const int64_t t = (int64_t)c * QT - 1 + lane;
    const bool ok = lane > 0 && lane < TQ && t < L;
    const int64_t idx = (b * L + (ok ? t : 0)) * H + h;
    pld = ok ? a.logdecay[idx] : 0.f;
    pga = ok ? a.gamma[idx] : 0.f;
    pbe = (ok && a.beta) ? a.beta[idx] : 0.f;
  };

  // ---- prologue -------------------------------------------------------------
  if (warp == 0) tc5::tmem_alloc(&sm.tmem, kTmemCols);
  if (ctrl_lead) {
    for (int i = 0; i < 4; ++i) tc5::mbar_init(&sm.mbar[i], 1);
    tc5::mbar_init(&sm.lmbar, 1);
    tc5::fence_mbar_init();
    sm.err = 0;
  }
  __syncthreads();
  if (ctrl_lead) {
    tc5::mbar_arrive_expect_tx(&sm.lmbar, chunk_bytes);
    if (ROT && has_theta) tma_theta(0);
    tma_bc(0, &tm.B, aB);
    tma_bc(0, &tm.C, aC);
    tma_x(0);
  }
  if (ctrl) {
    load_params(0);
    chunk_params<R>(sm.prm[0], pld, pbe, pga, lane);
    if (nC > 1) load_params(1);
  }
  const bool patch_row0 = a.bprev0 != nullptr || a.xprev0 != nullptr;
  if (ROT && tid < NH) sm.Phi[tid] = wrap_angle(a.angle0 ? a.angle0[bh * NH + tid] : 0.f);

  const int n_row = 32 * (warp & 3) + lane, cb = 32 * ((warp >> 2) & 1);
  float hs[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) hs[j] = 0.f;
  if (!ctrl && a.h0) {
    const float4* src = reinterpret_cast<const float4*>(a.h0 + (bh * NS + n_row) * PD + cb);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float4 v = src[j];
      hs[4 * j] = v.x; hs[4 * j + 1] = v.y; hs[4 * j + 2] = v.z; hs[4 * j + 3] = v.w;
    }
  }
  int kexp = 0;
  auto store_state_f16 = [&]() {
    float m = 0.f;
#pragma unroll
    for (int j = 0; j < 32; ++j) m = fmaxf(m, fabsf(hs[j]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) sm.hmax[warp] = m;
    asm volatile("bar.sync 2, %0;" ::"n"(32 * kCtrlWarp) : "memory");
    m = sm.hmax[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) m = fmaxf(m, sm.hmax[w]);
    kexp = 0;
    if (m > 0.f) {
      int e;
      frexpf(m, &e);
      kexp = min(max(14 - e, -100), 100);
    }
    const float sc = ldexpf(1.f, kexp);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint4 vh, vl;
      split_h2(sc * hs[8 * q + 0], sc * hs[8 * q + 1], vh.x, vl.x);
      split_h2(sc * hs[8 * q + 2], sc * hs[8 * q + 3], vh.y, vl.y);
      split_h2(sc * hs[8 * q + 4], sc * hs[8 * q + 5], vh.z, vl.z);
      split_h2(sc * hs[8 * q + 6], sc * hs[8 * q + 7], vh.w, vl.w);
      *reinterpret_cast<uint4*>(sm.Hs + off1(n_row, cb + 8 * q)) = vh;
      *reinterpret_cast<uint4*>(sm.Hs + NS * 128 + off1(n_row, cb + 8 * q)) = vl;
    }
  };
  if (!ctrl) store_state_f16();
  tc5::fence_proxy_async();
  tc5::fence_before_sync();
  __syncthreads();
  tc5::fence_after_sync();
  const uint32_t tmem = sm.tmem;
  const uint32_t tlane = (uint32_t)(32 * (warp & 3)) << 16;

  // ---- chunk walk -------------------------------------------------------------
  for (int c = 0; c < nC; ++c) {
    const int64_t tbase = (int64_t)c * QT - 1;
    const uint32_t par = (uint32_t)(c & 1);
    const MParams& P = sm.prm[c & 1];
    uint8_t* const Xs = sm.X[c & 1];
    const uint32_t aX = aX0 + (uint32_t)(c & 1) * (2 * kAtom);
    if (tid == 0 && !tc5::mbar_wait(&sm.lmbar, par, kWaitLimitNs)) sm.err = 1;
    tc5::fence_before_sync();
    __syncthreads();  // S1
    tc5::fence_after_sync();
    if (sm.err) {
      (void)tc5::mbar_wait(&sm.lmbar, par, kWaitLimitNs);
      if (c > 0) (void)tc5::mbar_wait(&sm.mbar[2], par ^ 1u, kWaitLimitNs);
      break;
    }

    if (ctrl) {
      // ===================== control warp ======================================
      if (ctrl_lead && c + 1 < nC) {
        tc5::mbar_arrive_expect_tx(&sm.lmbar, chunk_bytes);
        tma_x(c + 1);
      }
      if (c + 1 < nC) {
        chunk_params<R>(sm.prm[(c + 1) & 1], pld, pbe, pga, lane);
        if (c + 2 < nC) load_params(c + 2);
      }
      const uint64_t dC = tc5::desc_sw128(aC, 16, 1024), dB = tc5::desc_sw128(aB, 16, 1024);
      const uint64_t dBmh = tc5::desc_sw128(aB, 2 * kAtom, 1024);
      const uint64_t dBml = tc5::desc_sw128(aB + kAtom, 2 * kAtom, 1024);
      const uint64_t dWXh = tc5::desc_sw128(aWX, kAtom, 1024);
      const uint64_t dWXl = tc5::desc_sw128(aWX + kAtom, kAtom, 1024);
      const uint64_t dHh = tc5::desc_sw128(aH, kAtom, 1024);
      const uint64_t dHl = tc5::desc_sw128(aH + NS * 128, kAtom, 1024);
      const uint64_t dXh = tc5::desc_sw128(aX, kAtom, 1024);
      const uint64_t dXl = tc5::desc_sw128(aX + kAtom, kAtom, 1024);
      const uint64_t dMh = tc5::desc_sw128(aM, 16, 1024);
      const uint64_t dMl = tc5::desc_sw128(aM + kAtom, 16, 1024);
      constexpr uint64_t kLo = kAtom >> 4;
      __syncthreads();  // S3: operands ready; the angles are consumed
      if (ctrl_lead) {
        tc5::fence_after_sync();
        if (c + 1 < nC && ROT && has_theta) tma_theta(c + 1);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint64_t ko = (uint64_t)(((j >> 2) * 2 * kAtom + (j & 3) * 32) >> 4);
          tc5::mma_bf16(tmem + kColG, dC + ko, dB + ko, kIdescG, j > 0);
          tc5::mma_bf16(tmem + kColG, dC + ko, dB + ko + kLo, kIdescG, true);
          tc5::mma_bf16(tmem + kColG, dC + ko + kLo, dB + ko, kIdescG, true);
        }
        tc5::commit(&sm.mbar[0]);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint64_t k = (uint64_t)(j * (2048 >> 4));
          tc5::mma_bf16(tmem + kColS, dBmh + k, dWXh + k, kIdescS, j > 0);
          tc5::mma_bf16(tmem + kColS, dBmh + k, dWXl + k, kIdescS, true);
          tc5::mma_bf16(tmem + kColS, dBml + k, dWXh + k, kIdescS, true);
        }
        tc5::commit(&sm.mbar[3]);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint64_t ko = (uint64_t)(((j >> 2) * 2 * kAtom + (j & 3) * 32) >> 4);
          const uint64_t k = (uint64_t)(j * (2048 >> 4));
          tc5::mma_bf16(tmem + kColY1, dC + ko, dHh + k, kIdescY, j > 0);
          tc5::mma_bf16(tmem + kColY1, dC + ko, dHl + k, kIdescY, true);
          tc5::mma_bf16(tmem + kColY1, dC + ko + kLo, dHh + k, kIdescY, true);
        }
        tc5::commit(&sm.mbar[1]);
        if (c + 1 < nC) {
          if (!tc5::mbar_wait(&sm.mbar[3], par, kWaitLimitNs)) sm.err = 1;
          tma_bc(c + 1, &tm.B, aB);
        }
      }
      __syncthreads();  // S4: M ready
      if (ctrl_lead) {
        tc5::fence_after_sync();
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint64_t km = (uint64_t)(j * (32 >> 4)), kx = (uint64_t)(j * (2048 >> 4));
          tc5::mma_bf16(tmem + kColY2, dMh + km, dXh + kx, kIdescY, j > 0);
          tc5::mma_bf16(tmem + kColY2, dMh + km, dXl + kx, kIdescY, true);
          tc5::mma_bf16(tmem + kColY2, dMl + km, dXh + kx, kIdescY, true);
        }
        tc5::commit(&sm.mbar[2]);
        if (c + 1 < nC) {
          if (!tc5::mbar_wait(&sm.mbar[1], par, kWaitLimitNs)) sm.err = 1;
          tma_bc(c + 1, &tm.C, aC);
        }
      }
      continue;
    }

    // ===================== compute warps (0..7) ===================================
    if (c == 0 && patch_row0) {
      // token 0 of chunk 0 is the cache's previous token (zero-filled by the copy)
      if (a.bprev0)
        for (int e = tid; e < NS * R; e += 32 * kCtrlWarp)
          *reinterpret_cast<float*>(sm.B + (e / (32 * R)) * kAtom + (e % (32 * R)) * 4) =
              a.bprev0[(b * G + g) * NS * R + e];
      if (a.xprev0)
        for (int e = tid; e < PD * R; e += 32 * kCtrlWarp)
          *reinterpret_cast<float*>(sm.X[0] + (e / (32 * R)) * kAtom + (e % (32 * R)) * 4) =
              a.xprev0[bh * PD * R + e];
    }

    // -- phase R1: absolute angle of every token row --------------------------------
    if (ROT && has_theta) {
      constexpr int SR = TQ / 4;
      const int pr = tid & 63, seg = tid >> 6;
      float v[SR];
      float run = 0.f;
#pragma unroll
      for (int k = 0; k < SR; ++k) {
        const int j = seg * SR + k;
        if (j > 0) run += sm.ang[j][pr];
        v[k] = run;
      }
      sm.segtot[seg][pr] = run;
      asm volatile("bar.sync 1, %0;" ::"n"(32 * kCtrlWarp) : "memory");
      float base = sm.Phi[pr];
      for (int s2 = 0; s2 < seg; ++s2) base += sm.segtot[s2][pr];
#pragma unroll
      for (int k = 0; k < SR; ++k) sm.ang[seg * SR + k][pr] = base + v[k];
      if (seg == 3) sm.nPhi[pr] = wrap_angle(base + v[SR - 1]);
    }
    asm volatile("bar.sync 1, %0;" ::"n"(32 * kCtrlWarp) : "memory");

    // -- phase R2: rotation and fp16 high / low parts, transposed in place -----------
    // B and C: warp task = (token j, half hf of N); lane = pair 32 hf + lane, whose raw
    // values sit in n-block 2 hf + (lane >= 16) at 8R (lane % 16) bytes into the token
#pragma unroll 1
    for (int k = warp; k < 2 * TQ; k += kCtrlWarp) {
      const int j = k >> 1, hf = k & 1;
      const uint32_t off =
          (uint32_t)((2 * hf + (lane >> 4)) * kAtom + j * RB + 8 * R * (lane & 15));
      float vb[2 * R], vc[2 * R];
      lds_f<R>(sm.B + off, vb);
      lds_f<R>(sm.C + off, vc);
      __syncwarp();
      float cs = 1.f, sn = 0.f;
      if (ROT) __sincosf(has_theta ? sm.ang[j][32 * hf + lane] : sm.Phi[32 * hf + lane], &sn, &cs);
      const uint32_t hi_atom = (uint32_t)(2 * hf) * kAtom;
#pragma unroll
      for (int rho = 0; rho < R; ++rho) {
        // (B, C) packed: re = (b_re, c_re), im = (b_im, c_im)
        float2 re = make_float2(vb[rho], vc[rho]), im = make_float2(vb[R + rho], vc[R + rho]);
        if (ROT) {
          const float2 c2 = make_float2(cs, cs), s2 = make_float2(sn, sn);
          const float2 re2 = __ffma2_rn(make_float2(-sn, -sn), im, __fmul2_rn(c2, re));
          const float2 im2 = __ffma2_rn(c2, im, __fmul2_rn(s2, re));
          re = re2;
          im = im2;
        }
        uint32_t bh_, bl_, ch_, cl_;
        split_h2(re.x, im.x, bh_, bl_);
        split_h2(re.y, im.y, ch_, cl_);
        const uint32_t o = hi_atom + off1(R * j + rho, 2 * lane);
        *reinterpret_cast<uint32_t*>(sm.B + o) = bh_;
        *reinterpret_cast<uint32_t*>(sm.B + o + kAtom) = bl_;
        *reinterpret_cast<uint32_t*>(sm.C + o) = ch_;
        *reinterpret_cast<uint32_t*>(sm.C + o + kAtom) = cl_;
      }
    }
    // X: warp task = token j; lane = columns p = 2 lane, 2 lane + 1 of the token's R rows
#pragma unroll 1
    for (int j = warp; j < TQ; j += kCtrlWarp) {
      const uint32_t off = (uint32_t)((lane >> 4) * kAtom + j * RB + 8 * R * (lane & 15));
      float vx[2 * R];
      lds_f<R>(Xs + off, vx);
      __syncwarp();
      const float we = P.wend[R * j];
#pragma unroll
      for (int rho = 0; rho < R; ++rho) {
        const float x0 = vx[rho], x1 = vx[R + rho];  // p = 2 lane, 2 lane + 1
        const uint32_t o = off1(R * j + rho, 2 * lane);
        uint32_t xh, xl, wh, wl;
        split_h2(x0, x1, xh, xl);
        split_h2(we * x0, we * x1, wh, wl);
        *reinterpret_cast<uint32_t*>(Xs + o) = xh;
        *reinterpret_cast<uint32_t*>(Xs + kAtom + o) = xl;
        *reinterpret_cast<uint32_t*>(sm.wx + o) = wh;
        *reinterpret_cast<uint32_t*>(sm.wx + kAtom + o) = wl;
      }
    }
    tc5::fence_proxy_async();
    __syncthreads();  // S3
    if (ROT && has_theta && tid >= 2 * NH && tid < 3 * NH) sm.Phi[tid - 2 * NH] = sm.nPhi[tid - 2 * NH];

    // -- phase G: masked Gram -> M (high and low parts) --------------------------------
    {
      const int cpar = warp >> 2;
      float wv[2][4];
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int t = 16 * (warp & 3) + (lane >> 2) + 8 * hf;
        const int kr = 2 * (warp & 3) + hf;
        const int jt = t / R;
        const float et = P.et[t];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int kc = 2 * q + cpar;
          const int s0 = 8 * kc + 2 * (lane & 3);
          float w = 0.f;
          if (kc < kr) {
            w = et * P.fs[fs_index(kr, s0)];
          } else if (kc == kr) {
            const int js = s0 / R;
            if (js < jt) w = ex2(P.cs2[t] - P.csn2[s0]) * P.cvec[s0];
            else if (js == jt) w = P.gam[t];
          }
          wv[hf][q] = w;
        }
      }
      if (!tc5::mbar_wait(&sm.mbar[0], par, kWaitLimitNs)) sm.err = 1;
      tc5::fence_after_sync();
      uint32_t gr[4][4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        tc5::ld_16x256b_x1(tmem + tlane + kColG + (uint32_t)(8 * (2 * q + cpar)), gr[q]);
      tc5::wait_ld();
      tc5::reg_after_ld(gr[0]);
      tc5::reg_after_ld(gr[1]);
      tc5::reg_after_ld(gr[2]);
      tc5::reg_after_ld(gr[3]);
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int t = 16 * (warp & 3) + (lane >> 2) + 8 * hf;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int s0 = 8 * (2 * q + cpar) + 2 * (lane & 3);
          uint32_t mh, ml;
          split_h2(__uint_as_float(gr[q][2 * hf]) * wv[hf][q],
                   __uint_as_float(gr[q][2 * hf + 1]) * wv[hf][q], mh, ml);
          *reinterpret_cast<uint32_t*>(sm.M + off1(t, s0)) = mh;
          *reinterpret_cast<uint32_t*>(sm.M + kAtom + off1(t, s0)) = ml;
        }
      }
    }
    tc5::fence_proxy_async();
    tc5::fence_before_sync();
    __syncthreads();  // S4

    // -- phase S + Y: the state update while M X is in flight, then the outputs
    // (staged in M's space, fp32) ------------------------------------------------------
    {
      if (!tc5::mbar_wait(&sm.mbar[1], par, kWaitLimitNs)) sm.err = 1;  // G, S and Y1 done
      tc5::fence_after_sync();
      const float isc = ldexpf(1.f, -kexp);  // the scale Y1 used
      {
        uint32_t sv[32];
        tc5::ld_32x32b_x32(tmem + tlane + kColS + (uint32_t)cb, sv);
        tc5::wait_ld();
        tc5::reg_after_ld(sv);
        const float2 eE2 = make_float2(P.eE, P.eE);
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const float2 hv = __ffma2_rn(eE2, make_float2(hs[j], hs[j + 1]),
                                       make_float2(__uint_as_float(sv[j]), __uint_as_float(sv[j + 1])));
          hs[j] = hv.x;
          hs[j + 1] = hv.y;
        }
        store_state_f16();  // Y1 has read the previous copy
      }
      if (!tc5::mbar_wait(&sm.mbar[2], par, kWaitLimitNs)) sm.err = 1;
      tc5::fence_after_sync();
      uint32_t y1[16], y2[16];
      tc5::ld_16x256b_x4(tmem + tlane + kColY1 + (uint32_t)cb, y1);
      tc5::ld_16x256b_x4(tmem + tlane + kColY2 + (uint32_t)cb, y2);
      tc5::wait_ld();
      tc5::reg_after_ld(y1);
      tc5::reg_after_ld(y2);
      const float2 D2 = make_float2(Dh, Dh);
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int r = 16 * (warp & 3) + (lane >> 2) + 8 * hf;
        const int j = r / R, rho = r % R;
        if (j > 0 && tbase + j < L) {
          const float2 er2 = make_float2(P.ecs[r] * isc, P.ecs[r] * isc);
          // element (token j, p, rank rho) of the chunk's Y at ((j 64 + p) R + rho)
          float* const ys = reinterpret_cast<float*>(sm.M) + j * 64 * R + rho;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int p = cb + 8 * q + 2 * (lane & 3);
            const float2 xv =
                __fadd2_rn(unpack_h2(*reinterpret_cast<const uint32_t*>(Xs + off1(r, p))),
                           unpack_h2(*reinterpret_cast<const uint32_t*>(Xs + kAtom + off1(r, p))));
            const float2 a1 = make_float2(__uint_as_float(y1[4 * q + 2 * hf]),
                                          __uint_as_float(y1[4 * q + 2 * hf + 1]));
            const float2 a2 = make_float2(__uint_as_float(y2[4 * q + 2 * hf]),
                                          __uint_as_float(y2[4 * q + 2 * hf + 1]));
            const float2 v = __ffma2_rn(D2, xv, __ffma2_rn(er2, a1, a2));
            ys[p * R] = v.x;
            ys[(p + 1) * R] = v.y;
          }
        }
      }
      asm volatile("bar.sync 3, %0;" ::"n"(32 * kCtrlWarp) : "memory");  // Y staged
      // each token's (p, rank) run is 256 R contiguous bytes in HBM
#pragma unroll
      for (int gi = tid; gi < TQ * 16 * R; gi += 32 * kCtrlWarp) {
        const int j = gi / (16 * R), w = gi % (16 * R);
        const int64_t t = tbase + j;
        if (j > 0 && t < L)
          *reinterpret_cast<uint4*>(Yg8 + ((b * L + t) * H + h) * (int64_t)(PD * R * 4) + w * 16) =
              *reinterpret_cast<const uint4*>(sm.M + j * 2 * RB + w * 16);
      }
    }
    tc5::fence_proxy_async();
  }

  // ---- outputs of the last token, TMEM release ---------------------------------
  if (sm.err) {
    if (tid == 0) atomicAdd(&g_mimo32_wait_timeouts, 1u);
  } else if (!ctrl) {
    if (a.hT) {
      float4* dst = reinterpret_cast<float4*>(a.hT + (bh * NS + n_row) * PD + cb);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        dst[j] = make_float4(hs[4 * j], hs[4 * j + 1], hs[4 * j + 2], hs[4 * j + 3]);
    }
    if (a.angleT && tid < NH)
      a.angleT[bh * NH + tid] = ROT ? sm.Phi[tid] : (a.angle0 ? a.angle0[bh * NH + tid] : 0.f);
    if (a.xprevT)
      for (int e = tid; e < PD * R; e += 32 * kCtrlWarp)
        a.xprevT[bh * PD * R + e] = Xg[((b * L + L - 1) * H + h) * PD * R + e];
    if (a.bprevT && h % (H / G) == 0)
      for (int e = tid; e < NS * R; e += 32 * kCtrlWarp)
        a.bprevT[(b * G + g) * NS * R + e] = Bg[((b * L + L - 1) * G + g) * NS * R + e];
  }
  tc5::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc5::tmem_dealloc(tmem, kTmemCols);
}

bool encode(CUtensorMap* m, const void* base, const cuuint64_t* dims, const cuuint64_t* strides,
            const cuuint32_t* box) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = tensor_map_encoder();
  if (!fn) return false;
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int R, bool ROT>
cudaError_t launch_r32(const FwdArgs& a, cudaStream_t s) {
  MMaps32 tm;
  memset(&tm, 0, sizeof(tm));
  const cuuint64_t L = (cuuint64_t)a.L, b = (cuuint64_t)a.b, H = (cuuint64_t)a.H,
                   G = (cuuint64_t)a.G;
  const cuuint32_t TQ = Q / R;
  const cuuint64_t dB[4] = {(cuuint64_t)NS * R, G, L, b};
  const cuuint64_t sB[3] = {(cuuint64_t)NS * R * 4, G * NS * R * 4, L * G * NS * R * 4};
  const cuuint64_t dX[4] = {(cuuint64_t)PD * R, H, L, b};
  const cuuint64_t sX[3] = {(cuuint64_t)PD * R * 4, H * PD * R * 4, L * H * PD * R * 4};
  const cuuint32_t box[4] = {32u * R, 1, TQ, 1};
  bool ok = encode(&tm.B, a.B, dB, sB, box) && encode(&tm.C, a.C, dB, sB, box) &&
            encode(&tm.X, a.X, dX, sX, box);
  if (ok && a.theta) {
    const cuuint64_t dT[4] = {NH, H, L, b};
    const cuuint64_t sT[3] = {NH * 4, H * NH * 4, L * H * NH * 4};
    const cuuint32_t boxT[4] = {NH, 1, TQ, 1};
    ok = encode(&tm.theta, a.theta, dT, sT, boxT);
  }
  if (!ok) return cudaErrorInvalidValue;
  const size_t smem = sizeof(MSmem32) + 1024;
  cudaError_t e = cudaFuncSetAttribute(fwd_chunk_mimo32_kernel<R, ROT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  fwd_chunk_mimo32_kernel<R, ROT><<<(unsigned)(a.b * a.H), kThreads, smem, s>>>(a, tm);
  return cudaGetLastError();
}

template <int R>
cudaError_t launch_rank32(const FwdArgs& a, cudaStream_t s) {
  if (a.theta != nullptr || a.angle0 != nullptr) return launch_r32<R, true>(a, s);
  return launch_r32<R, false>(a, s);
}

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

bool fwd_chunk_mimo32_supported(const FwdArgs& a, int64_t R) {
  return !a.bf16 && a.N == NS && a.P == PD && a.L > 0 && (R == 2 || R == 4 || R == 8) &&
         a.x_tok_stride == 0 && a.Bbias == nullptr && a.Cbias == nullptr &&
         a.theta16 == nullptr && al16(a.X) && al16(a.B) && al16(a.C) && al16(a.Y) &&
         al16(a.theta) && al16(a.h0) && al16(a.hT);
}

cudaError_t launch_fwd_chunk_mimo32(const FwdArgs& a, int64_t R, cudaStream_t s) {
  if (a.b * a.H == 0) return cudaSuccess;
  switch (R) {
    case 2: return launch_rank32<2>(a, s);
    case 4: return launch_rank32<4>(a, s);
    case 8: return launch_rank32<8>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t read_and_clear_mimo32_wait_timeouts(unsigned int* count) {
  const unsigned int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(count, g_mimo32_wait_timeouts, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_mimo32_wait_timeouts, &zero, sizeof(unsigned int));
}

}  // namespace m3ssd
