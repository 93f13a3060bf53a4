// Chunked forward of the Mamba-3 SISO scan for fp32 X, B, C, Y on the sm_100a
// tensor cores, for N = 128, P = 64, accurate to about 2^-22 of each product.
//
// The chunk algebra, the per-(b, h) CTA with its control warp, the four
// products G = Cbar Bbar^T, S = Bbar^T (W_end o X), Y1 = Cbar h 2^k and
// Y2 = (W o G) X with their mbarriers, and the state kept in fp32 registers for
// the whole sequence are those of the bf16 chunked forward ("TorchMamba"
// README, "Math notes", M3 SISO; the chunk layout and mask are described
// there).  What differs is precision: every operand v of every product is held
// as two fp16 parts, hi = fp16(v) and lo = fp16(v - hi), and each product is
// the sum of three tensor-core MMAs hi.hi + hi.lo + lo.hi (fp32 accumulation
// in TMEM).  The dropped lo.lo term and the rounding of lo leave about 2^-22 of
// each term for values in fp16's normal range, with an absolute floor near
// 2^-25 below it; the state copy h 2^k is scaled by a power of two from its
// largest element as in the bf16 kernel, the other operands are not scaled.
//
// Shared memory: the fp32 inputs arrive by TMA in boxes of 32 columns, each
// placed where its rows' fp16 parts go: the raw boxes of columns 0-31, 32-63,
// 64-95 and 96-127 of B (or C) sit in the high atom 0, low atom 0, high atom 1
// and low atom 1 of the operand tile, so one row's 512 raw bytes are exactly
// that row's high and low bytes, and a warp that reads a whole row before
// writing converts it in place (the same for the two 32-column boxes of X).
// One CTA per SM (about 170 KB of shared memory).
#include <cuda.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <cstring>

#include "chunk_common.cuh"
#include "common.cuh"
#include "internal.h"
#include "tc5.cuh"

namespace m3ssd {

__device__ unsigned int g_chunk32_wait_timeouts;

namespace {

using namespace chunk;

constexpr int kCtrlWarp = 8;
constexpr int kThreads = 32 * (kCtrlWarp + 1);
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColG = 0, kColY1 = 64, kColY2 = 128, kColS = 192;
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr uint32_t kIdescG = tc5::idesc_f16(64, 64, false, false);
constexpr uint32_t kIdescY = tc5::idesc_f16(64, 64, false, true);
constexpr uint32_t kIdescS = tc5::idesc_f16(128, 64, true, true);

struct Smem32 {
  union {
    float theta[Q][NH];        // raw theta of the chunk (phase R1 only)
    uint8_t wx[2 * kAtom];     // W_end o X: high atom, low atom
  } u;
  uint8_t B[4 * kAtom];        // raw boxes, then Bbar: high atom 0, low 0, high 1, low 1
  uint8_t C[4 * kAtom];        // the same for C
  uint8_t X[2][2 * kAtom];     // raw boxes, then X: high atom, low atom (chunks c, c+1)
  uint8_t M[2 * kAtom];        // masked Gram: high, low
  uint8_t Hs[2 * NS * 128];    // h 2^k: high (128 rows of 128 B), low
  float hmax[8];
  ChunkParams prm[2];
  float segtot[8][NH];
  float Phi[NH];
  float nPhi[NH];
  uint64_t mbar[4];            // G done; Y1 (and S) done; Y2 done; S done
  uint64_t lmbar;
  uint32_t tmem;
  uint32_t err;
};
static_assert(sizeof(Smem32) + 1024 <= 232448, "one CTA per SM");


struct TmaMaps32 {
  CUtensorMap theta;  // fp32 (pair, head, token, batch), box 64 x 1 x 64 x 1
  CUtensorMap B;      // fp32 (n, group, token, batch), box 32 x 1 x 64 x 1
  CUtensorMap C;
  CUtensorMap X;      // fp32 (p, head, token, batch), box 32 x 1 x 64 x 1
};

template <bool ROT>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_chunk32_kernel(FwdArgs a, const __grid_constant__ TmaMaps32 tm) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw_addr = tc5::saddr(smem_raw);
  Smem32& sm = *reinterpret_cast<Smem32*>(smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool ctrl = warp == kCtrlWarp;
  const bool ctrl_lead = tid == kCtrlWarp * 32;
  const int64_t H = a.H, L = a.L, G = a.G;
  const int64_t bh = blockIdx.x;
  const int64_t b = bh / H, h = bh % H, g = h / (H / G);
  const int nC = (int)((L + QT - 1) / QT);
  const float* Xg = static_cast<const float*>(a.X);
  const float* Bg = static_cast<const float*>(a.B);
  float* Yg = static_cast<float*>(a.Y);
  const float Dh = a.D ? a.D[h] : 0.f;
  const uint32_t aB = tc5::saddr(sm.B), aC = tc5::saddr(sm.C);
  const uint32_t aX0 = tc5::saddr(sm.X[0]);
  const uint32_t aM = tc5::saddr(sm.M), aH = tc5::saddr(sm.Hs);
  const uint32_t aWX = tc5::saddr(sm.u.wx);
  const uint32_t aT = tc5::saddr(&sm.u.theta[0][0]);
  float* const Y_seq = Yg + (b * L * H + h) * PD;
  const int64_t xstride_t = H * PD;
  const bool has_theta = a.theta != nullptr;
  const uint32_t chunk_bytes = (ROT && has_theta ? 16384u : 0u) + 2u * 4u * kAtom + 2u * kAtom;
  auto tma_theta = [&](int c) {
    tc5::tma_load_4d(aT, &tm.theta, &sm.lmbar, 0, (int)h, c * QT - 1, (int)b);
  };
  auto tma_bc = [&](int c, const CUtensorMap* map, uint32_t base) {
#pragma unroll
    for (int k = 0; k < 4; ++k)
      tc5::tma_load_4d(base + (uint32_t)k * kAtom, map, &sm.lmbar, 32 * k, (int)g, c * QT - 1,
                       (int)b);
  };
  auto tma_x = [&](int c) {
    const uint32_t base = aX0 + (uint32_t)(c & 1) * (2 * kAtom);
    tc5::tma_load_4d(base, &tm.X, &sm.lmbar, 0, (int)h, c * QT - 1, (int)b);
    tc5::tma_load_4d(base + kAtom, &tm.X, &sm.lmbar, 32, (int)h, c * QT - 1, (int)b);
  };
  float pld[2], pbe[2], pga[2];
  auto load_params = [&](int c) {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int r = lane + 32 * k;
      const int64_t t = (int64_t)c * QT - 1 + r;
      const bool ok = r > 0 && t < L;
      const int64_t idx = (b * L + (ok ? t : 0)) * H + h;
      pld[k] = ok ? a.logdecay[idx] : 0.f;
      pga[k] = ok ? a.gamma[idx] : 0.f;
      pbe[k] = (ok && a.beta) ? a.beta[idx] : 0.f;
    }
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
    chunk_params(sm.prm[0], pld, pbe, pga, lane, 0.f);
    if (nC > 1) load_params(1);
  }
  const bool patch_row0 = a.bprev0 != nullptr || a.xprev0 != nullptr;
  if (ROT && tid < NH) sm.Phi[tid] = wrap_angle(a.angle0 ? a.angle0[bh * NH + tid] : 0.f);

  // state fragment (compute warps): row n = 32 (warp % 4) + lane, columns cb .. cb + 31
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
    const ChunkParams& P = sm.prm[c & 1];
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
        chunk_params(sm.prm[(c + 1) & 1], pld, pbe, pga, lane, 0.f);
        if (c + 2 < nC) load_params(c + 2);
      }
      // K-major Cbar, Bbar: high atoms 16 KB apart, low atom 8 KB after its high one;
      // MN-major Bbar (S's A operand): the same atoms; X, W_end o X, h: high, then low
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
      constexpr uint64_t kLo = kAtom >> 4;  // low atom after its high one (descriptor units)
      __syncthreads();  // S3
      if (ctrl_lead) {
        tc5::fence_after_sync();
        // G = Cbar Bbar^T: hi.hi + hi.lo + lo.hi, K = 128 in 8 steps
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint64_t ko = (uint64_t)(((j >> 2) * 2 * kAtom + (j & 3) * 32) >> 4);
          tc5::mma_bf16(tmem + kColG, dC + ko, dB + ko, kIdescG, j > 0);
          tc5::mma_bf16(tmem + kColG, dC + ko, dB + ko + kLo, kIdescG, true);
          tc5::mma_bf16(tmem + kColG, dC + ko + kLo, dB + ko, kIdescG, true);
        }
        tc5::commit(&sm.mbar[0]);
        // S = Bbar^T (W_end o X), K = 64 source rows
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint64_t k = (uint64_t)(j * (2048 >> 4));
          tc5::mma_bf16(tmem + kColS, dBmh + k, dWXh + k, kIdescS, j > 0);
          tc5::mma_bf16(tmem + kColS, dBmh + k, dWXl + k, kIdescS, true);
          tc5::mma_bf16(tmem + kColS, dBml + k, dWXh + k, kIdescS, true);
        }
        tc5::commit(&sm.mbar[3]);
        // Y1 = Cbar h 2^k, K = 128
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
        // Y2 = M X, K = 64 source rows
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
          if (ROT && has_theta) tma_theta(c + 1);
        }
      }
      continue;
    }

    // ===================== compute warps (0..7) ===================================
    if (c == 0 && patch_row0) {
      // row 0 of chunk 0 is the cache's previous token (zero-filled by the copy)
      if (tid < NS && a.bprev0)
        *reinterpret_cast<float*>(sm.B + (tid >> 5) * kAtom + (tid & 31) * 4) =
            a.bprev0[(b * G + g) * NS + tid];
      if (tid < PD && a.xprev0)
        *reinterpret_cast<float*>(sm.X[0] + (tid >> 5) * kAtom + (tid & 31) * 4) =
            a.xprev0[bh * PD + tid];
    }

    // -- phase R1: chunk-local angle sums; thread (lane, warp) owns pairs lane and
    // lane + 32 in rows 8 warp .. 8 warp + 7 ------------------------------------------
    float2 psi[8];
    if (ROT) {
      float2 run = make_float2(0.f, 0.f);
      if (has_theta) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          if (warp > 0 || k > 0) {
            const int r = 8 * warp + k;
            run = __fadd2_rn(run, make_float2(sm.u.theta[r][lane], sm.u.theta[r][lane + 32]));
          }
          psi[k] = run;
        }
      } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) psi[k] = run;
      }
      sm.segtot[warp][lane] = run.x;
      sm.segtot[warp][lane + 32] = run.y;
    }
    asm volatile("bar.sync 1, %0;" ::"n"(32 * kCtrlWarp) : "memory");  // S2

    // -- phase R2: rotation and fp16 high / low parts, in place --------------------
    {
      float2 base = make_float2(0.f, 0.f);
      if (ROT) {
        base = make_float2(sm.Phi[lane], sm.Phi[lane + 32]);
        for (int s2 = 0; s2 < warp; ++s2)
          base = __fadd2_rn(base, make_float2(sm.segtot[s2][lane], sm.segtot[s2][lane + 32]));
      }
      // lane's columns in atom A (A = 0, 1): 64 A + 2 lane, + 1, raw in box 2A + (lane >= 16)
      const uint32_t roff = (uint32_t)((lane >> 4) * kAtom + (lane & 15) * 8);
#pragma unroll 2
      for (int k = 0; k < 8; ++k) {
        const int r = 8 * warp + k;
        float2 rb[2], rc[2];
#pragma unroll
        for (int A = 0; A < 2; ++A) {
          const uint32_t o = (uint32_t)(2 * A) * kAtom + roff + (uint32_t)r * 128;
          rb[A] = *reinterpret_cast<const float2*>(sm.B + o);
          rc[A] = *reinterpret_cast<const float2*>(sm.C + o);
        }
        __syncwarp();  // the row's raw bytes are read before any part is written
#pragma unroll
        for (int A = 0; A < 2; ++A) {
          // (B, C) pairs packed together: re = (b_re, c_re), im = (b_im, c_im)
          float2 re = make_float2(rb[A].x, rc[A].x), im = make_float2(rb[A].y, rc[A].y);
          if (ROT) {
            const float ang = (A == 0 ? psi[k].x + base.x : psi[k].y + base.y);
            float sn, cs;
            __sincosf(ang, &sn, &cs);
            const float2 c2 = make_float2(cs, cs), s2 = make_float2(sn, sn);
            const float2 re2 = __ffma2_rn(make_float2(-sn, -sn), im, __fmul2_rn(c2, re));
            const float2 im2 = __ffma2_rn(c2, im, __fmul2_rn(s2, re));
            re = re2;
            im = im2;
          }
          uint32_t bh_, bl_, ch_, cl_;
          split_h2(re.x, im.x, bh_, bl_);
          split_h2(re.y, im.y, ch_, cl_);
          const uint32_t oh = (uint32_t)(2 * A) * kAtom + off1(r, 2 * lane);
          *reinterpret_cast<uint32_t*>(sm.B + oh) = bh_;
          *reinterpret_cast<uint32_t*>(sm.B + oh + kAtom) = bl_;
          *reinterpret_cast<uint32_t*>(sm.C + oh) = ch_;
          *reinterpret_cast<uint32_t*>(sm.C + oh + kAtom) = cl_;
        }
      }
      {  // X in high / low parts (in place) and W_end o X: row tid / 4, columns 16 (tid % 4) ..
        const int r = tid >> 2, qd = tid & 3;
        const float we = P.wend[r];
        const float4* src =
            reinterpret_cast<const float4*>(Xs + (qd >> 1) * kAtom + r * 128 + (qd & 1) * 64);
        float xv[16];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float4 v = src[j];
          xv[4 * j] = v.x; xv[4 * j + 1] = v.y; xv[4 * j + 2] = v.z; xv[4 * j + 3] = v.w;
        }
        __syncwarp();
#pragma unroll
        for (int hq = 0; hq < 2; ++hq) {  // 16-byte chunks 2 qd, 2 qd + 1 of the row
          const int ch = 2 * qd + hq;
          const uint32_t o = (uint32_t)(r * 128 + ((ch ^ (r & 7)) << 4));
          uint4 xh, xl, wh, wl;
          split_h2(xv[8 * hq + 0], xv[8 * hq + 1], xh.x, xl.x);
          split_h2(xv[8 * hq + 2], xv[8 * hq + 3], xh.y, xl.y);
          split_h2(xv[8 * hq + 4], xv[8 * hq + 5], xh.z, xl.z);
          split_h2(xv[8 * hq + 6], xv[8 * hq + 7], xh.w, xl.w);
          split_h2(we * xv[8 * hq + 0], we * xv[8 * hq + 1], wh.x, wl.x);
          split_h2(we * xv[8 * hq + 2], we * xv[8 * hq + 3], wh.y, wl.y);
          split_h2(we * xv[8 * hq + 4], we * xv[8 * hq + 5], wh.z, wl.z);
          split_h2(we * xv[8 * hq + 6], we * xv[8 * hq + 7], wh.w, wl.w);
          *reinterpret_cast<uint4*>(Xs + o) = xh;
          *reinterpret_cast<uint4*>(Xs + kAtom + o) = xl;
          *reinterpret_cast<uint4*>(sm.u.wx + o) = wh;
          *reinterpret_cast<uint4*>(sm.u.wx + kAtom + o) = wl;
        }
      }
      if (ROT && warp == 7) {
        sm.nPhi[lane] = wrap_angle(psi[7].x + base.x);
        sm.nPhi[lane + 32] = wrap_angle(psi[7].y + base.y);
      }
    }
    tc5::fence_proxy_async();
    __syncthreads();  // S3
    if (ROT && tid >= 2 * NH && tid < 3 * NH) sm.Phi[tid - 2 * NH] = sm.nPhi[tid - 2 * NH];

    // -- phase G: masked Gram -> M (high and low parts) ------------------------------
    {
      const int cpar = warp >> 2;
      float wv[2][4][2];
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int t = 16 * (warp & 3) + (lane >> 2) + 8 * hf;
        const int kr = 2 * (warp & 3) + hf;
        const float et = P.et[t];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int kc = 2 * q + cpar;
          const int s0 = 8 * kc + 2 * (lane & 3);
          float w0 = 0.f, w1 = 0.f;
          if (kc < kr) {
            const float2 f = *reinterpret_cast<const float2*>(&P.fs[fs_index(kr, s0)]);
            w0 = et * f.x;
            w1 = et * f.y;
          } else if (kc == kr) {
            const float cst = P.cs2[t];
            if (s0 < t) w0 = ex2(cst - P.cs2[s0 + 1]) * P.cvec[s0];
            else if (s0 == t) w0 = P.gam[t];
            if (s0 + 1 < t) w1 = ex2(cst - P.cs2[s0 + 2]) * P.cvec[s0 + 1];
            else if (s0 + 1 == t) w1 = P.gam[t];
          }
          wv[hf][q][0] = w0;
          wv[hf][q][1] = w1;
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
          split_h2(__uint_as_float(gr[q][2 * hf]) * wv[hf][q][0],
                   __uint_as_float(gr[q][2 * hf + 1]) * wv[hf][q][1], mh, ml);
          *reinterpret_cast<uint32_t*>(sm.M + off1(t, s0)) = mh;
          *reinterpret_cast<uint32_t*>(sm.M + kAtom + off1(t, s0)) = ml;
        }
      }
    }
    tc5::fence_proxy_async();
    tc5::fence_before_sync();
    __syncthreads();  // S4

    // -- phase Y + S: outputs and the state update ---------------------------------
    {
      if (!tc5::mbar_wait(&sm.mbar[2], par, kWaitLimitNs)) sm.err = 1;
      tc5::fence_after_sync();
      uint32_t y1[16], y2[16];
      tc5::ld_16x256b_x4(tmem + tlane + kColY1 + (uint32_t)cb, y1);
      tc5::ld_16x256b_x4(tmem + tlane + kColY2 + (uint32_t)cb, y2);
      tc5::wait_ld();
      tc5::reg_after_ld(y1);
      tc5::reg_after_ld(y2);
      const float2 D2 = make_float2(Dh, Dh);
      const float isc = ldexpf(1.f, -kexp);
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int r = 16 * (warp & 3) + (lane >> 2) + 8 * hf;
        const int64_t t = tbase + r;
        if (r > 0 && t < L) {
          const float2 er2 = make_float2(P.ecs[r] * isc, P.ecs[r] * isc);
          float* yrow = Y_seq + t * xstride_t;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int p = cb + 8 * q + 2 * (lane & 3);
            const float2 xh = unpack_h2(*reinterpret_cast<const uint32_t*>(Xs + off1(r, p)));
            const float2 xl =
                unpack_h2(*reinterpret_cast<const uint32_t*>(Xs + kAtom + off1(r, p)));
            const float2 xv = __fadd2_rn(xh, xl);
            const float2 a1 = make_float2(__uint_as_float(y1[4 * q + 2 * hf]),
                                          __uint_as_float(y1[4 * q + 2 * hf + 1]));
            const float2 a2 = make_float2(__uint_as_float(y2[4 * q + 2 * hf]),
                                          __uint_as_float(y2[4 * q + 2 * hf + 1]));
            *reinterpret_cast<float2*>(yrow + p) = __ffma2_rn(D2, xv, __ffma2_rn(er2, a1, a2));
          }
        }
      }
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
      store_state_f16();
    }
    tc5::fence_proxy_async();
  }

  // ---- outputs of the last token, TMEM release ---------------------------------
  if (sm.err) {
    if (tid == 0) atomicAdd(&g_chunk32_wait_timeouts, 1u);
  } else if (!ctrl) {
    if (a.hT) {
      float4* dst = reinterpret_cast<float4*>(a.hT + (bh * NS + n_row) * PD + cb);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        dst[j] = make_float4(hs[4 * j], hs[4 * j + 1], hs[4 * j + 2], hs[4 * j + 3]);
    }
    if (a.angleT && tid < NH)
      a.angleT[bh * NH + tid] = ROT ? sm.Phi[tid] : (a.angle0 ? a.angle0[bh * NH + tid] : 0.f);
    if (a.xprevT && tid < PD) a.xprevT[bh * PD + tid] = Xg[((b * L + L - 1) * H + h) * PD + tid];
    if (a.bprevT && h % (H / G) == 0 && tid < NS)
      a.bprevT[(b * G + g) * NS + tid] = Bg[((b * L + L - 1) * G + g) * NS + tid];
  }
  tc5::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc5::tmem_dealloc(tmem, kTmemCols);
}

template <bool ROT>
cudaError_t launch_variant32(const FwdArgs& a, cudaStream_t s) {
  TmaMaps32 tm;
  memset(&tm, 0, sizeof(tm));
  const uint64_t L = (uint64_t)a.L, b = (uint64_t)a.b, H = (uint64_t)a.H, G = (uint64_t)a.G;
  bool ok = encode_map(&tm.B, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, a.B, NS, G, L, b, 4, 32,
                       CU_TENSOR_MAP_SWIZZLE_NONE) &&
            encode_map(&tm.C, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, a.C, NS, G, L, b, 4, 32,
                       CU_TENSOR_MAP_SWIZZLE_NONE) &&
            encode_map(&tm.X, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, a.X, PD, H, L, b, 4, 32,
                       CU_TENSOR_MAP_SWIZZLE_NONE);
  if (ok && a.theta)
    ok = encode_map(&tm.theta, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, a.theta, NH, H, L, b, 4, NH,
                    CU_TENSOR_MAP_SWIZZLE_NONE);
  if (!ok) return cudaErrorInvalidValue;
  const size_t smem = sizeof(Smem32) + 1024;
  cudaError_t e = cudaFuncSetAttribute(fwd_chunk32_kernel<ROT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  fwd_chunk32_kernel<ROT><<<(unsigned)(a.b * a.H), kThreads, smem, s>>>(a, tm);
  return cudaGetLastError();
}

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

bool fwd_chunk32_supported(const FwdArgs& a) {
  return !a.bf16 && a.N == NS && a.P == PD && a.L > 0 && (a.chunk == 0 || a.chunk == Q) &&
         a.x_tok_stride == 0 && a.theta16 == nullptr && a.Bbias == nullptr &&
         a.Cbias == nullptr && al16(a.X) && al16(a.B) && al16(a.C) && al16(a.Y) &&
         al16(a.theta) && al16(a.h0) && al16(a.hT);
}

cudaError_t launch_fwd_chunk32(const FwdArgs& a, cudaStream_t s) {
  if (a.b * a.H == 0) return cudaSuccess;
  if (a.theta != nullptr || a.angle0 != nullptr) return launch_variant32<true>(a, s);
  return launch_variant32<false>(a, s);
}

cudaError_t read_and_clear_chunk32_wait_timeouts(unsigned int* count) {
  const unsigned int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(count, g_chunk32_wait_timeouts, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_chunk32_wait_timeouts, &zero, sizeof(unsigned int));
}

}  // namespace m3ssd
