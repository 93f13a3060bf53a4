// Chunked bf16 forward of the Mamba-3 MIMO scan at rank R = 2, 4 or 8 on the
// sm_100a tensor cores (tcgen05 MMA, TMEM accumulators), for N = 128, P = 64.
//
// The MIMO recurrence ("TorchMamba" README, "Math notes", MIMO; table "Models",
// Mamba-3 MIMO row) replaces the SISO outer product Bbar x^T by the rank-R sum
// sum_rho Bbar_{t,rho} x_{t,rho}^T on the shared (N, P) state and reads R output
// columns y_{t,rho} = Cbar_{t,rho}^T h_t + D x_{t,rho}.  Unrolled over a chunk it
// is the SISO chunk algebra with one source row per (token, rank): the Gram
// Cbar Bbar^T, the masked Gram times X, the state product Bbar^T (W_end o X) and
// the state-to-output product Cbar h keep their 64-row tile shapes when a chunk
// holds 64 / R tokens (the pages' "chunked C_MIMO = C_SISO / R"), and the
// trapezoid weight W(t, u) of a token pair fills an R x R block of the mask.
//
// Chunk layout.  64 rows; row R j + rho holds chunk-local token j and rank rho.
// Token 0 is the token just before the chunk (the carry-in of the beta term),
// tokens 1 .. 64/R - 1 are the chunk's own.  With the per-token weights of the
// SISO kernel (decay sums cs_j, gamma_j, cvec_j = gamma_j alpha_{j+1} +
// beta_{j+1}, gamma_0 := 0) the mask is
//     W(row r, row s) = gamma_j                          if token(s) = token(r) = j
//                     = exp(cs_j - cs_{k+1}) cvec_k      if token(s) = k < j = token(r)
//                     = 0                                otherwise,
// so every rank of a token sees every rank of the same token through gamma.
//
// The per-(b, h) CTA, its control warp, the four products with their mbarriers,
// the fp16 operands, the power-of-two scaled fp16 copy of the state and the
// bounded waits are those of the SISO chunked forward.  What differs is the
// data movement: X, B and C keep the rank axis innermost in HBM ((b,L,H,P,R) and
// (b,L,G,N,R)), and a 5-D tensor map lands each token's R x 64 values in exactly
// the bytes its R operand rows occupy (R 128-byte rows), so the rotation and the
// fp16 conversion transpose them in place, one warp per token (and per half of
// N for B and C).  Y leaves through the masked-Gram tile, staged there in the
// (token, p, rank) order of HBM once the tensor core has read the mask, and is
// written with 16-byte coalesced stores.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <cstring>

#include "common.cuh"
#include "internal.h"
#include "mimo_chunk.cuh"
#include "tc5.cuh"

namespace m3ssd {

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

// Number of bounded device-side waits of this kernel that ran out.
__device__ unsigned int g_mimo_chunk_wait_timeouts;

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

typedef __nv_bfloat16 bf16;


struct MSmem {
  float ang[32][NH];           // theta of the chunk's token rows, then their absolute angles
  uint8_t wx[Q * 128];         // W_end o X (fp16)
  uint8_t B[2 * kAtom];        // raw B (token, n, rank), then the Bbar rows (fp16)
  uint8_t C[2 * kAtom];        // the same for C
  uint8_t X[2][Q * 128];       // raw X (token, p, rank), then the X rows (fp16)
  uint8_t M[Q * 128];          // masked Gram (fp16); after Y2, the chunk's Y in HBM order
  uint8_t Hs[NS * 128];        // fp16 copy of h 2^k
  float hmax[8];
  MParams prm[2];
  float segtot[4][NH];
  float Phi[NH];
  float nPhi[NH];
  uint64_t mbar[4];            // G done; Y1 (and S) done; Y2 done; S done
  uint64_t lmbar;
  uint32_t tmem;
  uint32_t err;
};
static_assert(2 * (sizeof(MSmem) + 1024 + 1024) <= 233472, "two CTAs per SM");


// 4R bytes of shared memory (R words) into registers, in 16- or 8-byte pieces.
template <int R>
__device__ __forceinline__ void lds_words(const uint8_t* p, uint32_t (&w)[R]) {
  if constexpr (R == 2) {
    const uint2 v = *reinterpret_cast<const uint2*>(p);
    w[0] = v.x; w[1] = v.y;
  } else {
#pragma unroll
    for (int i = 0; i < R / 4; ++i) {
      const uint4 v = reinterpret_cast<const uint4*>(p)[i];
      w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
    }
  }
}

struct MMaps {
  CUtensorMap theta;  // fp32 (pair, head, token, batch), box 64 x 1 x (64/R) x 1
  CUtensorMap B;      // bf16 (16R, N/16, group, token, batch), box 16R x 4 x 1 x (64/R) x 1
  CUtensorMap C;      // same as B
  CUtensorMap X;      // bf16 (16R, P/16, head, token, batch), box 16R x 4 x 1 x (64/R) x 1
};

template <int R, bool ROT>
__global__ void __launch_bounds__(kThreads, 2)
    fwd_chunk_mimo_kernel(FwdArgs a, const __grid_constant__ MMaps tm) {
  static_assert(R == 2 || R == 4 || R == 8, "rank");
  constexpr int TQ = Q / R;   // token rows per chunk (with the carry-in)
  constexpr int QT = TQ - 1;  // new tokens per chunk
  constexpr int RB = 128 * R; // bytes of one token's R rows (and of its raw values per half of N)
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw_addr = tc5::saddr(smem_raw);
  MSmem& sm = *reinterpret_cast<MSmem*>(smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool ctrl = warp == kCtrlWarp;
  const bool ctrl_lead = tid == kCtrlWarp * 32;
  const int64_t H = a.H, L = a.L, G = a.G;
  const int64_t bh = blockIdx.x;
  const int64_t b = bh / H, h = bh % H, g = h / (H / G);
  const int nC = (int)((L + QT - 1) / QT);
  const bf16* Xg = static_cast<const bf16*>(a.X);
  const bf16* Bg = static_cast<const bf16*>(a.B);
  uint8_t* const Yg8 = static_cast<uint8_t*>(a.Y);
  const float Dh = a.D ? a.D[h] : 0.f;
  const uint32_t aB = tc5::saddr(sm.B), aC = tc5::saddr(sm.C);
  const uint32_t aX0 = tc5::saddr(sm.X[0]);
  const uint32_t aM = tc5::saddr(sm.M), aH = tc5::saddr(sm.Hs);
  const uint32_t aWX = tc5::saddr(sm.wx);
  const uint32_t aT = tc5::saddr(&sm.ang[0][0]);
  const bool has_theta = a.theta != nullptr;
  const uint32_t chunk_bytes =
      (ROT && has_theta ? (uint32_t)(TQ * NH * 4) : 0u) + 4u * kAtom + (uint32_t)(Q * 128);
  auto tma_theta = [&](int c) {
    tc5::tma_load_4d(aT, &tm.theta, &sm.lmbar, 0, (int)h, c * QT - 1, (int)b);
  };
  auto tma_bc = [&](int c, const CUtensorMap* map, uint32_t base) {
    tc5::tma_load_5d(base, map, &sm.lmbar, 0, 0, (int)g, c * QT - 1, (int)b);
    tc5::tma_load_5d(base + kAtom, map, &sm.lmbar, 0, 4, (int)g, c * QT - 1, (int)b);
  };
  auto tma_x = [&](int c) {
    tc5::tma_load_5d(aX0 + (uint32_t)(c & 1) * (Q * 128), &tm.X, &sm.lmbar, 0, 0, (int)h,
                     c * QT - 1, (int)b);
  };
  // the control warp keeps logdecay / beta / gamma of token lane of the next chunk
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

  // state fragment (compute warps): row n = 32 (warp % 4) + lane, columns cb .. cb + 31.
  // Between chunks the fp32 state lives in TMEM, in the state product's columns:
  // before chunk c they hold exp(cs of c's last token) h, onto which S accumulates.
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
  auto store_state_f16 = [&](const float (&hs)[32]) {
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
      uint4 v;
      v.x = pack_h2(sc * hs[8 * q + 0], sc * hs[8 * q + 1]);
      v.y = pack_h2(sc * hs[8 * q + 2], sc * hs[8 * q + 3]);
      v.z = pack_h2(sc * hs[8 * q + 4], sc * hs[8 * q + 5]);
      v.w = pack_h2(sc * hs[8 * q + 6], sc * hs[8 * q + 7]);
      *reinterpret_cast<uint4*>(sm.Hs + off1(n_row, cb + 8 * q)) = v;
    }
  };
  if (!ctrl) store_state_f16(hs);
  tc5::fence_proxy_async();
  tc5::fence_before_sync();
  __syncthreads();
  tc5::fence_after_sync();
  const uint32_t tmem = sm.tmem;
  const uint32_t tlane = (uint32_t)(32 * (warp & 3)) << 16;
  auto store_state_tmem = [&](const float (&hv)[32], float scale) {
    uint32_t w[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) w[j] = __float_as_uint(scale * hv[j]);
    tc5::st_32x32b_x32(tmem + tlane + kColS + (uint32_t)cb, w);
    tc5::wait_st();
  };
  if (!ctrl) store_state_tmem(hs, sm.prm[0].eE);

  // ---- chunk walk -------------------------------------------------------------
  for (int c = 0; c < nC; ++c) {
    const int64_t tbase = (int64_t)c * QT - 1;  // token of chunk-local token 0
    const uint32_t par = (uint32_t)(c & 1);
    const MParams& P = sm.prm[c & 1];
    uint8_t* const Xs = sm.X[c & 1];
    const uint32_t aX = aX0 + (uint32_t)(c & 1) * (Q * 128);
    if (tid == 0 && !tc5::mbar_wait(&sm.lmbar, par, kWaitLimitNs)) sm.err = 1;
    tc5::fence_before_sync();
    __syncthreads();  // S1: this chunk's inputs are in shared memory
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
      const uint64_t dH = tc5::desc_sw128(aH, kAtom, 1024), dX = tc5::desc_sw128(aX, kAtom, 1024);
      const uint64_t dBm = tc5::desc_sw128(aB, kAtom, 1024), dWX = tc5::desc_sw128(aWX, kAtom, 1024);
      const uint64_t dM = tc5::desc_sw128(aM, 16, 1024);
      __syncthreads();  // S3: Cbar, Bbar, X, W_end o X ready; the angles are consumed
      if (ctrl_lead) {
        tc5::fence_after_sync();
        if (c + 1 < nC && ROT && has_theta) tma_theta(c + 1);
        // G = Cbar Bbar^T (both K-major), K = 128
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint64_t ko = (uint64_t)(((j >> 2) * kAtom + (j & 3) * 32) >> 4);
          tc5::mma_bf16(tmem + kColG, dC + ko, dB + ko, kIdescG, j > 0);
        }
        tc5::commit(&sm.mbar[0]);
        // S = Bbar^T (W_end o X), K = 64 source rows
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint64_t kofs = (uint64_t)(j * (2048 >> 4));
          tc5::mma_bf16(tmem + kColS, dBm + kofs, dWX + kofs, kIdescS, true);
        }
        tc5::commit(&sm.mbar[3]);
        // Y1 = Cbar h 2^k
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint64_t ko = (uint64_t)(((j >> 2) * kAtom + (j & 3) * 32) >> 4);
          tc5::mma_bf16(tmem + kColY1, dC + ko, dH + (uint64_t)(j * (2048 >> 4)), kIdescY, j > 0);
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
        for (int j = 0; j < 4; ++j)
          tc5::mma_bf16(tmem + kColY2, dM + (uint64_t)(j * (32 >> 4)),
                        dX + (uint64_t)(j * (2048 >> 4)), kIdescY, j > 0);
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
          *reinterpret_cast<bf16*>(sm.B + (e / (64 * R)) * kAtom + (e % (64 * R)) * 2) =
              __float2bfloat16_rn(a.bprev0[(b * G + g) * NS * R + e]);
      if (a.xprev0)
        for (int e = tid; e < PD * R; e += 32 * kCtrlWarp)
          *reinterpret_cast<bf16*>(sm.X[0] + e * 2) = __float2bfloat16_rn(a.xprev0[bh * PD * R + e]);
    }

    // -- phase R1: absolute angle of every token row ------------------------------
    // Thread (pair tid % 64, segment tid / 64) sums theta over its segment of TQ/4
    // token rows (token 0 adds nothing: its angle is the chunk's start angle).
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

    // -- phase R2: rotation, fp16 conversion and transposition in place -----------
    // B and C: warp task = (token j, half hf of N); lane = pair 32 hf + lane, whose
    // raw values [n = 2i][rank], [n = 2i + 1][rank] sit at lane 4R bytes into the
    // token's 128R bytes, which become the token's R Bbar rows (columns 2 lane,
    // 2 lane + 1 of the half's atom).
#pragma unroll 1
    for (int k = warp; k < 2 * TQ; k += kCtrlWarp) {
      const int j = k >> 1, hf = k & 1;
      const uint32_t off = (uint32_t)(hf * kAtom + j * RB + lane * 4 * R);
      uint32_t wb[R], wc[R];
      lds_words<R>(sm.B + off, wb);
      lds_words<R>(sm.C + off, wc);
      __syncwarp();
      float cs = 1.f, sn = 0.f;
      if (ROT) __sincosf(has_theta ? sm.ang[j][32 * hf + lane] : sm.Phi[32 * hf + lane], &sn, &cs);
      const float2 c2 = make_float2(cs, cs), s2 = make_float2(sn, sn), ns2 = make_float2(-sn, -sn);
      uint8_t* const bdst = sm.B + hf * kAtom;
      uint8_t* const cdst = sm.C + hf * kAtom;
#pragma unroll
      for (int q = 0; q < R / 2; ++q) {  // ranks 2q, 2q + 1
        float2 bre = unpack_bf16(wb[q]), bim = unpack_bf16(wb[R / 2 + q]);
        float2 cre = unpack_bf16(wc[q]), cim = unpack_bf16(wc[R / 2 + q]);
        if (ROT) {
          const float2 bre2 = __ffma2_rn(ns2, bim, __fmul2_rn(c2, bre));
          const float2 bim2 = __ffma2_rn(c2, bim, __fmul2_rn(s2, bre));
          const float2 cre2 = __ffma2_rn(ns2, cim, __fmul2_rn(c2, cre));
          const float2 cim2 = __ffma2_rn(c2, cim, __fmul2_rn(s2, cre));
          bre = bre2; bim = bim2; cre = cre2; cim = cim2;
        }
        const int r0 = R * j + 2 * q;
        *reinterpret_cast<uint32_t*>(bdst + off1(r0, 2 * lane)) = pack_h2(bre.x, bim.x);
        *reinterpret_cast<uint32_t*>(bdst + off1(r0 + 1, 2 * lane)) = pack_h2(bre.y, bim.y);
        *reinterpret_cast<uint32_t*>(cdst + off1(r0, 2 * lane)) = pack_h2(cre.x, cim.x);
        *reinterpret_cast<uint32_t*>(cdst + off1(r0 + 1, 2 * lane)) = pack_h2(cre.y, cim.y);
      }
    }
    // X: warp task = token j; lane = columns p = 2 lane, 2 lane + 1 of the token's R rows
#pragma unroll 1
    for (int j = warp; j < TQ; j += kCtrlWarp) {
      const uint32_t off = (uint32_t)(j * RB + lane * 4 * R);
      uint32_t wx[R];
      lds_words<R>(Xs + off, wx);
      __syncwarp();
      const float we = P.wend[R * j];
#pragma unroll
      for (int q = 0; q < R / 2; ++q) {
        const float2 x0 = unpack_bf16(wx[q]);          // p = 2 lane, ranks 2q, 2q + 1
        const float2 x1 = unpack_bf16(wx[R / 2 + q]);  // p = 2 lane + 1
        const int r0 = R * j + 2 * q;
        const uint32_t o0 = off1(r0, 2 * lane), o1 = off1(r0 + 1, 2 * lane);
        *reinterpret_cast<uint32_t*>(Xs + o0) = pack_h2(x0.x, x1.x);
        *reinterpret_cast<uint32_t*>(Xs + o1) = pack_h2(x0.y, x1.y);
        *reinterpret_cast<uint32_t*>(sm.wx + o0) = pack_h2(we * x0.x, we * x1.x);
        *reinterpret_cast<uint32_t*>(sm.wx + o1) = pack_h2(we * x0.y, we * x1.y);
      }
    }
    tc5::fence_proxy_async();
    __syncthreads();  // S3
    if (ROT && has_theta && tid >= 2 * NH && tid < 3 * NH) sm.Phi[tid - 2 * NH] = sm.nPhi[tid - 2 * NH];

    // -- phase G: masked Gram -> M ----------------------------------------------------
    {
      const int cpar = warp >> 2;
      float wv[2][4];  // rows s0 and s0 + 1 belong to one token (R even): one weight
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
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int t = 16 * (warp & 3) + (lane >> 2) + 8 * hf;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int s0 = 8 * (2 * q + cpar) + 2 * (lane & 3);
          *reinterpret_cast<uint32_t*>(sm.M + off1(t, s0)) =
              pack_h2(__uint_as_float(gr[q][2 * hf]) * wv[hf][q],
                      __uint_as_float(gr[q][2 * hf + 1]) * wv[hf][q]);
        }
      }
    }
    tc5::fence_proxy_async();
    tc5::fence_before_sync();
    __syncthreads();  // S4: M ready

    // -- phase S + Y: the state update while M X is in flight, then the outputs
    // (staged in M's space) ---------------------------------------------------------
    {
      if (!tc5::mbar_wait(&sm.mbar[1], par, kWaitLimitNs)) sm.err = 1;  // G, S and Y1 done
      tc5::fence_after_sync();
      const float isc = ldexpf(1.f, -kexp);  // the scale Y1 used
      {
        uint32_t sv[32];
        tc5::ld_32x32b_x32(tmem + tlane + kColS + (uint32_t)cb, sv);
        tc5::wait_ld();
        tc5::reg_after_ld(sv);
        float hv[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) hv[j] = __uint_as_float(sv[j]);
        store_state_f16(hv);  // Y1 has read the previous copy
        if (c + 1 < nC) store_state_tmem(hv, sm.prm[(c + 1) & 1].eE);
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
          bf16* const ys = reinterpret_cast<bf16*>(sm.M + j * RB) + rho;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int p = cb + 8 * q + 2 * (lane & 3);
            const float2 xv = unpack_h2(*reinterpret_cast<const uint32_t*>(Xs + off1(r, p)));
            const float2 a1 = make_float2(__uint_as_float(y1[4 * q + 2 * hf]),
                                          __uint_as_float(y1[4 * q + 2 * hf + 1]));
            const float2 a2 = make_float2(__uint_as_float(y2[4 * q + 2 * hf]),
                                          __uint_as_float(y2[4 * q + 2 * hf + 1]));
            const float2 v = __ffma2_rn(D2, xv, __ffma2_rn(er2, a1, a2));
            ys[p * R] = __float2bfloat16_rn(v.x);
            ys[(p + 1) * R] = __float2bfloat16_rn(v.y);
          }
        }
      }
      asm volatile("bar.sync 3, %0;" ::"n"(32 * kCtrlWarp) : "memory");  // Y staged
      // the chunk's tokens are contiguous (token, p, rank) runs of 128R bytes in HBM
#pragma unroll
      for (int gi = tid; gi < TQ * 8 * R; gi += 32 * kCtrlWarp) {
        const int j = gi / (8 * R), w = gi % (8 * R);
        const int64_t t = tbase + j;
        if (j > 0 && t < L)
          *reinterpret_cast<uint4*>(Yg8 + ((b * L + t) * H + h) * (int64_t)(PD * R * 2) + w * 16) =
              *reinterpret_cast<const uint4*>(sm.M + j * RB + w * 16);
      }
    }
    tc5::fence_proxy_async();
  }

  // ---- outputs of the last token, TMEM release ---------------------------------
  if (sm.err) {
    if (tid == 0) atomicAdd(&g_mimo_chunk_wait_timeouts, 1u);
  } else if (!ctrl) {
    if (a.hT) {  // after the last chunk TMEM holds h itself
      uint32_t sv[32];
      tc5::ld_32x32b_x32(tmem + tlane + kColS + (uint32_t)cb, sv);
      tc5::wait_ld();
      tc5::reg_after_ld(sv);
      float4* dst = reinterpret_cast<float4*>(a.hT + (bh * NS + n_row) * PD + cb);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        dst[j] = make_float4(__uint_as_float(sv[4 * j]), __uint_as_float(sv[4 * j + 1]),
                             __uint_as_float(sv[4 * j + 2]), __uint_as_float(sv[4 * j + 3]));
    }
    if (a.angleT && tid < NH)
      a.angleT[bh * NH + tid] = ROT ? sm.Phi[tid] : (a.angle0 ? a.angle0[bh * NH + tid] : 0.f);
    if (a.xprevT)
      for (int e = tid; e < PD * R; e += 32 * kCtrlWarp)
        a.xprevT[bh * PD * R + e] = __bfloat162float(Xg[((b * L + L - 1) * H + h) * PD * R + e]);
    if (a.bprevT && h % (H / G) == 0)
      for (int e = tid; e < NS * R; e += 32 * kCtrlWarp)
        a.bprevT[(b * G + g) * NS * R + e] =
            __bfloat162float(Bg[((b * L + L - 1) * G + g) * NS * R + e]);
  }
  tc5::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc5::tmem_dealloc(tmem, kTmemCols);
}

// A tiled tensor map with no swizzle (zero fill outside the tensor).
bool encode(CUtensorMap* m, CUtensorMapDataType dt, const void* base, cuuint32_t rank,
            const cuuint64_t* dims, const cuuint64_t* strides, const cuuint32_t* box) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = tensor_map_encoder();
  if (!fn) return false;
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return fn(m, dt, rank, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int R, bool ROT>
cudaError_t launch_r(const FwdArgs& a, cudaStream_t s) {
  MMaps tm;
  memset(&tm, 0, sizeof(tm));
  const cuuint64_t L = (cuuint64_t)a.L, b = (cuuint64_t)a.b, H = (cuuint64_t)a.H,
                   G = (cuuint64_t)a.G;
  const cuuint32_t TQ = Q / R;
  const cuuint64_t dB[5] = {16u * R, NS / 16, G, L, b};
  const cuuint64_t sB[4] = {32u * R, (cuuint64_t)NS * R * 2, G * NS * R * 2, L * G * NS * R * 2};
  const cuuint64_t dX[5] = {16u * R, PD / 16, H, L, b};
  const cuuint64_t sX[4] = {32u * R, (cuuint64_t)PD * R * 2, H * PD * R * 2, L * H * PD * R * 2};
  const cuuint32_t box[5] = {16u * R, 4, 1, TQ, 1};
  bool ok = encode(&tm.B, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.B, 5, dB, sB, box) &&
            encode(&tm.C, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.C, 5, dB, sB, box) &&
            encode(&tm.X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.X, 5, dX, sX, box);
  if (ok && a.theta) {
    const cuuint64_t dT[4] = {NH, H, L, b};
    const cuuint64_t sT[3] = {NH * 4, H * NH * 4, L * H * NH * 4};
    const cuuint32_t boxT[4] = {NH, 1, TQ, 1};
    ok = encode(&tm.theta, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, a.theta, 4, dT, sT, boxT);
  }
  if (!ok) return cudaErrorInvalidValue;
  const size_t smem = sizeof(MSmem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(fwd_chunk_mimo_kernel<R, ROT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  fwd_chunk_mimo_kernel<R, ROT><<<(unsigned)(a.b * a.H), kThreads, smem, s>>>(a, tm);
  return cudaGetLastError();
}

template <int R>
cudaError_t launch_rank(const FwdArgs& a, cudaStream_t s) {
  if (a.theta != nullptr || a.angle0 != nullptr) return launch_r<R, true>(a, s);
  return launch_r<R, false>(a, s);
}

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

bool fwd_chunk_mimo_supported(const FwdArgs& a, int64_t R) {
  return a.bf16 && a.N == NS && a.P == PD && a.L > 0 && (R == 2 || R == 4 || R == 8) &&
         a.x_tok_stride == 0 && a.Bbias == nullptr && a.Cbias == nullptr &&
         a.theta16 == nullptr && al16(a.X) && al16(a.B) && al16(a.C) && al16(a.Y) &&
         al16(a.theta) && al16(a.h0) && al16(a.hT);
}

cudaError_t launch_fwd_chunk_mimo(const FwdArgs& a, int64_t R, cudaStream_t s) {
  if (a.b * a.H == 0) return cudaSuccess;
  switch (R) {
    case 2: return launch_rank<2>(a, s);
    case 4: return launch_rank<4>(a, s);
    case 8: return launch_rank<8>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t read_and_clear_mimo_wait_timeouts(unsigned int* count) {
  const unsigned int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(count, g_mimo_chunk_wait_timeouts, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_mimo_chunk_wait_timeouts, &zero, sizeof(unsigned int));
}

}  // namespace m3ssd
