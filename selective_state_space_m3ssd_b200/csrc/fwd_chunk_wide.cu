// Chunked bf16 forward of the Mamba-3 SISO scan with chunks of Q = 128 or 256
// rows (T = Q / 64 sub-tiles), for N = 128, P = 64.
//
// The chunk length Q is the span of the intra-chunk quadratic form: within a
// chunk every pair of rows interacts through the masked Gram, across chunks
// only through the state ("TorchMamba" README, "Math notes", M2: chunkwise
// intra-quadratic with a factored inter-chunk carry).  Chunk row 0 is the token
// before the chunk (the beta term's carry-in), rows 1 .. Q-1 are the chunk's own
// tokens, and the mask and state weights are those of the 64-row kernel over the
// longer chunk (decay sums cs from the chunk start):
//     y_r   = exp(cs_r) Cbar_r^T h + sum_{u<=r} W(r,u) (Cbar_r^T Bbar_u) x_u + D x_r
//     h_end = exp(cs_end) h + sum_u W(end,u) Bbar_u x_u^T.
// The chunk is walked in sub-tiles of 64 rows.  Sub-tile i adds the Gram blocks
// G_ij = Cbar_i Bbar_j^T of every earlier sub-tile j of the chunk, so the Bbar
// and X of the chunk's sub-tiles stay in shared memory until the chunk ends.
// A block below the diagonal has a rank-one mask,
//     W(r,u) = exp(cs_r - m_i) . exp(m_i - cs_{u+1}) (gamma_u alpha_{u+1} + beta_{u+1}),
// m_i the decay sum at sub-tile i's first row (both factors at most 1), and the
// diagonal block keeps the 64-row kernel's factorised mask.  Y1 = Cbar_i h reads
// the chunk-start state for every sub-tile; S accumulates over the chunk in TMEM
// and the fp32 state is updated once per chunk.  Operands are fp16 as in the
// 64-row kernel (the state copy scaled by a power of two).  One CTA per SM
// (130 KB of shared memory at Q = 128, 203 KB at Q = 256; 512 TMEM columns).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <cstring>

#include "chunk_common.cuh"
#include "common.cuh"
#include "internal.h"
#include "tc5.cuh"

namespace m3ssd {

__device__ unsigned int g_wide_wait_timeouts;

namespace {

using namespace chunk;

constexpr int kCtrlWarp = 8;
constexpr int kThreads = 32 * (kCtrlWarp + 1);
constexpr uint32_t kTmemCols = 512;
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr uint32_t kIdescG = tc5::idesc_f16(64, 64, false, false);
constexpr uint32_t kIdescY = tc5::idesc_f16(64, 64, false, true);
constexpr uint32_t kIdescS = tc5::idesc_f16(128, 64, true, true);

// Per-chunk scalars for QW = 64 T rows (log2 units for the decay sums).
template <int T>
struct WParams {
  static constexpr int QW = 64 * T;
  float cs2[QW];     // cs_r log2(e), cs_0 = 0 at the carry-in row
  float ecs[QW];     // exp(cs_r)
  float cvec[QW];    // gamma_r alpha_{r+1} + beta_{r+1} (gamma of the last row)
  float wend[QW];    // W(QW - 1, r)
  float gam[QW];     // gamma_r
  float et[QW];      // exp(cs_r - cs at the row's 8-row block start)
  float arow[QW];    // exp(cs_r - cs at the row's sub-tile start)
  float fs[T][224];  // sub-tile i's diagonal-block factor table (as the 64-row kernel's)
  float bcol[32 * T * (T - 1)];  // sub-tile i's column factors for rows u < 64 i, at 32 i (i - 1) + u
  float eE;          // exp(cs_end)
  float pad[3];
};

template <int T>
struct WSmem {
  union {
    float theta[Q][NH];     // raw theta of the sub-tile (phase R1 only)
    uint8_t wx[Q * 128];    // W_end o X of the sub-tile (fp16)
  } u;
  uint8_t B[T][2 * kAtom];  // Bbar of every sub-tile of the chunk
  uint8_t C[2 * kAtom];     // Cbar of the current sub-tile
  uint8_t X[T][Q * 128];    // X of every sub-tile of the chunk (fp16)
  uint8_t M[T][Q * 128];    // masked Gram blocks of the current sub-tile's rows
  uint8_t Hs[NS * 128];     // fp16 copy of the chunk-start state h 2^k
  float hmax[8];
  WParams<T> prm[2];
  float segtot[8][NH];
  float Phi[NH];
  float nPhi[NH];
  uint64_t mbar[4];         // G done; Y1 (and S) done; Y2 done; S done
  uint64_t lmbar;
  uint32_t tmem;
  uint32_t err;
};

// The control warp: the scalars of one chunk from its per-row logdecay / beta /
// gamma (rows lane + 32 k; row 0 and rows past the end hold zeros).
template <int T>
__device__ __forceinline__ void wide_params(WParams<T>& P, const float (&pld)[2 * T],
                                            const float (&pbe)[2 * T], const float (&pga)[2 * T],
                                            int lane) {
  constexpr int R2 = 2 * T;
  float cs[R2];
  float carry = 0.f;
#pragma unroll
  for (int k = 0; k < R2; ++k) {
    float s = pld[k] * kLog2e;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float u = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += u;
    }
    cs[k] = s + carry;
    carry = __shfl_sync(0xffffffffu, cs[k], 31);
  }
  const float cs_end = carry;
#pragma unroll
  for (int k = 0; k < R2; ++k) {
    const int r = lane + 32 * k;
    // the next row: lane + 1 of the same group, or lane 0 of the next group
    const float ld_dn = __shfl_down_sync(0xffffffffu, pld[k], 1);
    const float be_dn = __shfl_down_sync(0xffffffffu, pbe[k], 1);
    const float cs_dn = __shfl_down_sync(0xffffffffu, cs[k], 1);
    const float ld_nx = k + 1 < R2 ? __shfl_sync(0xffffffffu, pld[k + 1 < R2 ? k + 1 : k], 0) : 0.f;
    const float be_nx = k + 1 < R2 ? __shfl_sync(0xffffffffu, pbe[k + 1 < R2 ? k + 1 : k], 0) : 0.f;
    const float cs_nx = k + 1 < R2 ? __shfl_sync(0xffffffffu, cs[k + 1 < R2 ? k + 1 : k], 0) : 0.f;
    const float ld_next = lane < 31 ? ld_dn : ld_nx;
    const float be_next = lane < 31 ? be_dn : be_nx;
    const float cs_next = lane < 31 ? cs_dn : cs_nx;
    const float blk8 = __shfl_sync(0xffffffffu, cs[k], lane & ~7);
    const float sub0 = __shfl_sync(0xffffffffu, cs[k & ~1], 0);  // row 64 (k / 2)
    P.cs2[r] = cs[k];
    P.ecs[r] = ex2(cs[k]);
    P.gam[r] = pga[k];
    P.et[r] = ex2(cs[k] - blk8);
    P.arow[r] = ex2(cs[k] - sub0);
    float cv;
    if (r < 64 * T - 1) {
      cv = pga[k] * ex2(ld_next * kLog2e) + be_next;
      P.wend[r] = ex2(cs_end - cs_next) * cv;
    } else {
      cv = pga[k];
      P.wend[r] = cv;
    }
    P.cvec[r] = cv;
    // the diagonal-block table of this row's sub-tile i = k / 2 (local row s)
    const int i = k >> 1, s = r - 64 * i;
#pragma unroll
    for (int k2 = 1; k2 < 8; ++k2) {
      const float mk = __shfl_sync(0xffffffffu, cs[2 * i + (k2 >= 4 ? 1 : 0)], (8 * k2) & 31);
      if (8 * k2 > s) P.fs[i][fs_index(k2, s)] = ex2(mk - cs_next) * cv;
    }
    // the column factors of every later sub-tile i2 > i
#pragma unroll
    for (int i2 = 1; i2 < T; ++i2) {
      const float mi = __shfl_sync(0xffffffffu, cs[2 * i2], 0);
      if (i2 > i) P.bcol[32 * i2 * (i2 - 1) + r] = ex2(mi - cs_next) * cv;
    }
  }
  if (lane == 0) P.eE = ex2(cs_end);
}

struct WMaps {
  CUtensorMap theta;
  CUtensorMap B;
  CUtensorMap C;
  CUtensorMap X;
};

template <int T, bool ROT>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_chunk_wide_kernel(FwdArgs a, const __grid_constant__ WMaps tm) {
  constexpr int QW = 64 * T, QTW = QW - 1;
  constexpr uint32_t kColY1 = 64 * T, kColY2 = 64 * T + 64, kColS = 64 * T + 128;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw_addr = tc5::saddr(smem_raw);
  WSmem<T>& sm =
      *reinterpret_cast<WSmem<T>*>(smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool ctrl = warp == kCtrlWarp;
  const bool ctrl_lead = tid == kCtrlWarp * 32;
  const int64_t H = a.H, L = a.L, G = a.G;
  const int64_t bh = blockIdx.x;
  const int64_t b = bh / H, h = bh % H, g = h / (H / G);
  const int nC = (int)((L + QTW - 1) / QTW);
  const int nS = nC * T;  // sub-tile steps
  const __nv_bfloat16* Xg = static_cast<const __nv_bfloat16*>(a.X);
  const __nv_bfloat16* Bg = static_cast<const __nv_bfloat16*>(a.B);
  __nv_bfloat16* Yg = static_cast<__nv_bfloat16*>(a.Y);
  const float Dh = a.D ? a.D[h] : 0.f;
  const uint32_t aC = tc5::saddr(sm.C), aH = tc5::saddr(sm.Hs);
  const uint32_t aWX = tc5::saddr(sm.u.wx);
  const uint32_t aT = tc5::saddr(&sm.u.theta[0][0]);
  __nv_bfloat16* const Y_seq = Yg + (b * L * H + h) * PD;
  const int64_t xstride_t = H * PD;
  const bool has_theta = a.theta != nullptr;
  const uint32_t step_bytes = (ROT && has_theta ? 16384u : 0u) + 2u * 16384u + 8192u;
  // token of row 0 of sub-tile step s (chunk s / T, sub-tile s % T)
  auto row0_token = [&](int s) { return (s / T) * QTW - 1 + 64 * (s % T); };
  auto tma_theta = [&](int s) {
    tc5::tma_load_4d(aT, &tm.theta, &sm.lmbar, 0, (int)h, row0_token(s), (int)b);
  };
  auto tma_b = [&](int s) {
    const uint32_t base = tc5::saddr(sm.B[s % T]);
    tc5::tma_load_4d(base, &tm.B, &sm.lmbar, 0, (int)g, row0_token(s), (int)b);
    tc5::tma_load_4d(base + kAtom, &tm.B, &sm.lmbar, 64, (int)g, row0_token(s), (int)b);
  };
  auto tma_c = [&](int s) {
    tc5::tma_load_4d(aC, &tm.C, &sm.lmbar, 0, (int)g, row0_token(s), (int)b);
    tc5::tma_load_4d(aC + kAtom, &tm.C, &sm.lmbar, 64, (int)g, row0_token(s), (int)b);
  };
  auto tma_x = [&](int s) {
    tc5::tma_load_4d(tc5::saddr(sm.X[s % T]), &tm.X, &sm.lmbar, 0, (int)h, row0_token(s), (int)b);
  };
  float pld[2 * T], pbe[2 * T], pga[2 * T];
  auto load_params = [&](int c) {
#pragma unroll
    for (int k = 0; k < 2 * T; ++k) {
      const int r = lane + 32 * k;
      const int64_t t = (int64_t)c * QTW - 1 + r;
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
    tc5::mbar_arrive_expect_tx(&sm.lmbar, step_bytes);
    if (ROT && has_theta) tma_theta(0);
    tma_b(0);
    tma_c(0);
    tma_x(0);
  }
  if (ctrl) {
    load_params(0);
    wide_params<T>(sm.prm[0], pld, pbe, pga, lane);
    if (nC > 1) load_params(1);
  }
  const float bp0 = (tid < NS && a.bprev0) ? a.bprev0[(b * G + g) * NS + tid] : 0.f;
  const float xp0 = (tid < PD && a.xprev0) ? a.xprev0[bh * PD + tid] : 0.f;
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
      uint4 v;
      v.x = pack_h2(sc * hs[8 * q + 0], sc * hs[8 * q + 1]);
      v.y = pack_h2(sc * hs[8 * q + 2], sc * hs[8 * q + 3]);
      v.z = pack_h2(sc * hs[8 * q + 4], sc * hs[8 * q + 5]);
      v.w = pack_h2(sc * hs[8 * q + 6], sc * hs[8 * q + 7]);
      *reinterpret_cast<uint4*>(sm.Hs + off1(n_row, cb + 8 * q)) = v;
    }
  };
  if (!ctrl) store_state_f16();
  tc5::fence_proxy_async();
  tc5::fence_before_sync();
  __syncthreads();
  tc5::fence_after_sync();
  const uint32_t tmem = sm.tmem;
  const uint32_t tlane = (uint32_t)(32 * (warp & 3)) << 16;

  // ---- sub-tile walk ------------------------------------------------------------
  for (int st = 0; st < nS; ++st) {
    const int c = st / T, i = st % T;
    const int64_t tbase = (int64_t)c * QTW - 1 + 64 * i;  // token of the sub-tile's row 0
    const uint32_t par = (uint32_t)(st & 1);
    const WParams<T>& P = sm.prm[c & 1];
    uint8_t* const Xs = sm.X[i];
    if (tid == 0 && !tc5::mbar_wait(&sm.lmbar, par, kWaitLimitNs)) sm.err = 1;
    tc5::fence_before_sync();
    __syncthreads();  // S1: the sub-tile's theta, B, C, X are in shared memory
    tc5::fence_after_sync();
    if (sm.err) {
      (void)tc5::mbar_wait(&sm.lmbar, par, kWaitLimitNs);
      if (st > 0) (void)tc5::mbar_wait(&sm.mbar[2], par ^ 1u, kWaitLimitNs);
      break;
    }

    if (ctrl) {
      // ===================== control warp ======================================
      const bool more = st + 1 < nS;
      const bool next_in_chunk = i + 1 < T;  // the next step's B and X slots are free now
      if (ctrl_lead && more) {
        tc5::mbar_arrive_expect_tx(&sm.lmbar, step_bytes);
        if (next_in_chunk) {
          tma_x(st + 1);
          tma_b(st + 1);
        }
      }
      if (i == 0 && c + 1 < nC) {
        wide_params<T>(sm.prm[(c + 1) & 1], pld, pbe, pga, lane);
        if (c + 2 < nC) load_params(c + 2);
      }
      const uint64_t dC = tc5::desc_sw128(aC, 16, 1024);
      const uint64_t dH = tc5::desc_sw128(aH, kAtom, 1024);
      const uint64_t dWX = tc5::desc_sw128(aWX, kAtom, 1024);
      __syncthreads();  // S3
      if (ctrl_lead) {
        tc5::fence_after_sync();
        // G_ij = Cbar_i Bbar_j^T for j = 0 .. i (TMEM columns 64 j ..)
        for (int j = 0; j <= i; ++j) {
          const uint64_t dB = tc5::desc_sw128(tc5::saddr(sm.B[j]), 16, 1024);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t ko = (uint64_t)(((kk >> 2) * kAtom + (kk & 3) * 32) >> 4);
            tc5::mma_bf16(tmem + (uint32_t)(64 * j), dC + ko, dB + ko, kIdescG, kk > 0);
          }
        }
        tc5::commit(&sm.mbar[0]);
        // S += Bbar_i^T (W_end o X_i)
        const uint64_t dBm = tc5::desc_sw128(tc5::saddr(sm.B[i]), kAtom, 1024);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t k = (uint64_t)(kk * (2048 >> 4));
          tc5::mma_bf16(tmem + kColS, dBm + k, dWX + k, kIdescS, i > 0 || kk > 0);
        }
        tc5::commit(&sm.mbar[3]);
        // Y1 = Cbar_i h 2^k (the chunk-start state)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t ko = (uint64_t)(((kk >> 2) * kAtom + (kk & 3) * 32) >> 4);
          tc5::mma_bf16(tmem + kColY1, dC + ko, dH + (uint64_t)(kk * (2048 >> 4)), kIdescY, kk > 0);
        }
        tc5::commit(&sm.mbar[1]);
      }
      __syncthreads();  // S4: the masked Gram blocks are ready
      if (ctrl_lead) {
        tc5::fence_after_sync();
        // Y2 = sum_j M_ij X_j
        for (int j = 0; j <= i; ++j) {
          const uint64_t dM = tc5::desc_sw128(tc5::saddr(sm.M[j]), 16, 1024);
          const uint64_t dX = tc5::desc_sw128(tc5::saddr(sm.X[j]), kAtom, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc5::mma_bf16(tmem + kColY2, dM + (uint64_t)(kk * (32 >> 4)),
                          dX + (uint64_t)(kk * (2048 >> 4)), kIdescY, j > 0 || kk > 0);
        }
        tc5::commit(&sm.mbar[2]);
        if (more) {
          if (next_in_chunk) {
            // C and theta (W_end o X's space) are free once Y1 (and S) are done
            if (!tc5::mbar_wait(&sm.mbar[1], par, kWaitLimitNs)) sm.err = 1;
          } else {
            // the next chunk's sub-tile 0 reuses slot 0, read by every product of this one
            if (!tc5::mbar_wait(&sm.mbar[2], par, kWaitLimitNs)) sm.err = 1;
            tma_x(st + 1);
            tma_b(st + 1);
          }
          tma_c(st + 1);
          if (ROT && has_theta) tma_theta(st + 1);
        }
      }
      continue;
    }

    // ===================== compute warps (0..7) ===================================
    if (st == 0 && patch_row0) {
      if (tid < NS) *reinterpret_cast<__nv_bfloat16*>(sm.B[0] + off2(0, tid)) = __float2bfloat16_rn(bp0);
      if (tid < PD) *reinterpret_cast<__nv_bfloat16*>(sm.X[0] + off1(0, tid)) = __float2bfloat16_rn(xp0);
    }

    // -- phase R1: sub-tile-local angle sums (row 0 of sub-tile 0 is the carry-in) --
    float2 psi[8];
    if (ROT) {
      float2 run = make_float2(0.f, 0.f);
      if (has_theta) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          if (i > 0 || warp > 0 || k > 0)
            run = __fadd2_rn(run, *reinterpret_cast<const float2*>(&sm.u.theta[8 * warp + k][2 * lane]));
          psi[k] = run;
        }
      } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) psi[k] = run;
      }
      *reinterpret_cast<float2*>(&sm.segtot[warp][2 * lane]) = run;
    }
    asm volatile("bar.sync 1, %0;" ::"n"(32 * kCtrlWarp) : "memory");  // S2

    // -- phase R2: rotation into the absolute frame; X and W_end o X in fp16 -------
    {
      uint8_t* const Bs = sm.B[i];
      float2 base = make_float2(0.f, 0.f);
      if (ROT) {
        base = *reinterpret_cast<const float2*>(&sm.Phi[2 * lane]);
        for (int s2 = 0; s2 < warp; ++s2)
          base = __fadd2_rn(base, *reinterpret_cast<const float2*>(&sm.segtot[s2][2 * lane]));
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int r = 8 * warp + k;
        const uint32_t o = off2(r, 4 * lane);
        uint2* pb = reinterpret_cast<uint2*>(Bs + o);
        uint2* pc = reinterpret_cast<uint2*>(sm.C + o);
        const uint2 bw2 = *pb, cw2 = *pc;
        float2 bre = make_float2(__uint_as_float(bw2.x << 16), __uint_as_float(bw2.y << 16));
        float2 bim = make_float2(__uint_as_float(bw2.x & 0xffff0000u),
                                 __uint_as_float(bw2.y & 0xffff0000u));
        float2 cre = make_float2(__uint_as_float(cw2.x << 16), __uint_as_float(cw2.y << 16));
        float2 cim = make_float2(__uint_as_float(cw2.x & 0xffff0000u),
                                 __uint_as_float(cw2.y & 0xffff0000u));
        if (ROT) {
          const float2 ang = __fadd2_rn(psi[k], base);
          float s0, c0, s1, c1;
          __sincosf(ang.x, &s0, &c0);
          __sincosf(ang.y, &s1, &c1);
          const float2 cr = make_float2(c0, c1), sr = make_float2(s0, s1);
          const float2 nsr = make_float2(-s0, -s1);
          const float2 bre2 = __ffma2_rn(nsr, bim, __fmul2_rn(cr, bre));
          const float2 bim2 = __ffma2_rn(cr, bim, __fmul2_rn(sr, bre));
          const float2 cre2 = __ffma2_rn(nsr, cim, __fmul2_rn(cr, cre));
          const float2 cim2 = __ffma2_rn(cr, cim, __fmul2_rn(sr, cre));
          bre = bre2; bim = bim2; cre = cre2; cim = cim2;
        }
        *pb = make_uint2(pack_h2(bre.x, bim.x), pack_h2(bre.y, bim.y));
        *pc = make_uint2(pack_h2(cre.x, cim.x), pack_h2(cre.y, cim.y));
      }
      {
        const int r = tid >> 2;
        const float we = P.wend[64 * i + r];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int ch = 2 * (tid & 3) + q;
          const uint32_t o = (uint32_t)(r * 128 + ((ch ^ (r & 7)) << 4));
          uint4* px = reinterpret_cast<uint4*>(Xs + o);
          const uint4 xw = *px;
          const uint32_t w4[4] = {xw.x, xw.y, xw.z, xw.w};
          float xv[8];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            xv[2 * j] = __uint_as_float(w4[j] << 16);
            xv[2 * j + 1] = __uint_as_float(w4[j] & 0xffff0000u);
          }
          *px = make_uint4(pack_h2(xv[0], xv[1]), pack_h2(xv[2], xv[3]), pack_h2(xv[4], xv[5]),
                           pack_h2(xv[6], xv[7]));
          *reinterpret_cast<uint4*>(sm.u.wx + o) =
              make_uint4(pack_h2(we * xv[0], we * xv[1]), pack_h2(we * xv[2], we * xv[3]),
                         pack_h2(we * xv[4], we * xv[5]), pack_h2(we * xv[6], we * xv[7]));
        }
      }
      if (ROT && warp == 7) {
        const float2 pend = __fadd2_rn(psi[7], base);
        sm.nPhi[2 * lane] = wrap_angle(pend.x);
        sm.nPhi[2 * lane + 1] = wrap_angle(pend.y);
      }
    }
    tc5::fence_proxy_async();
    __syncthreads();  // S3
    if (ROT && tid >= 2 * NH && tid < 3 * NH) sm.Phi[tid - 2 * NH] = sm.nPhi[tid - 2 * NH];

    // -- phase G: masked Gram blocks M_ij, j = 0 .. i --------------------------------
    {
      const int cpar = warp >> 2;
      if (!tc5::mbar_wait(&sm.mbar[0], par, kWaitLimitNs)) sm.err = 1;
      tc5::fence_after_sync();
      for (int j = 0; j <= i; ++j) {
        float wv[2][4][2];
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int tl = 16 * (warp & 3) + (lane >> 2) + 8 * hf;  // row in the sub-tile
          const int t = 64 * i + tl;                             // row in the chunk
          const int kr = 2 * (warp & 3) + hf;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int kc = 2 * q + cpar;
            const int s0 = 8 * kc + 2 * (lane & 3);
            float w0 = 0.f, w1 = 0.f;
            if (j < i) {
              const float ar = P.arow[t];
              const float2 f =
                  *reinterpret_cast<const float2*>(&P.bcol[32 * i * (i - 1) + 64 * j + s0]);
              w0 = ar * f.x;
              w1 = ar * f.y;
            } else if (kc < kr) {
              const float et = P.et[t];
              const float2 f = *reinterpret_cast<const float2*>(&P.fs[i][fs_index(kr, s0)]);
              w0 = et * f.x;
              w1 = et * f.y;
            } else if (kc == kr) {
              const int u = 64 * i + s0;
              const float cst = P.cs2[t];
              if (s0 < tl) w0 = ex2(cst - P.cs2[u + 1]) * P.cvec[u];
              else if (s0 == tl) w0 = P.gam[t];
              if (s0 + 1 < tl) w1 = ex2(cst - P.cs2[u + 2]) * P.cvec[u + 1];
              else if (s0 + 1 == tl) w1 = P.gam[t];
            }
            wv[hf][q][0] = w0;
            wv[hf][q][1] = w1;
          }
        }
        uint32_t gr[4][4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
          tc5::ld_16x256b_x1(tmem + tlane + (uint32_t)(64 * j + 8 * (2 * q + cpar)), gr[q]);
        tc5::wait_ld();
        tc5::reg_after_ld(gr[0]);
        tc5::reg_after_ld(gr[1]);
        tc5::reg_after_ld(gr[2]);
        tc5::reg_after_ld(gr[3]);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int tl = 16 * (warp & 3) + (lane >> 2) + 8 * hf;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int s0 = 8 * (2 * q + cpar) + 2 * (lane & 3);
            *reinterpret_cast<uint32_t*>(sm.M[j] + off1(tl, s0)) =
                pack_h2(__uint_as_float(gr[q][2 * hf]) * wv[hf][q][0],
                        __uint_as_float(gr[q][2 * hf + 1]) * wv[hf][q][1]);
          }
        }
      }
    }
    tc5::fence_proxy_async();
    tc5::fence_before_sync();
    __syncthreads();  // S4

    // -- phase Y (+ the state update at the chunk's last sub-tile) -----------------
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
        const int rl = 16 * (warp & 3) + (lane >> 2) + 8 * hf;
        const int r = 64 * i + rl;
        const int64_t t = tbase + rl;
        if (r > 0 && t < L) {
          const float2 er2 = make_float2(P.ecs[r] * isc, P.ecs[r] * isc);
          __nv_bfloat16* yrow = Y_seq + t * xstride_t;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int p = cb + 8 * q + 2 * (lane & 3);
            const float2 xv = unpack_h2(*reinterpret_cast<const uint32_t*>(Xs + off1(rl, p)));
            const float2 a1 = make_float2(__uint_as_float(y1[4 * q + 2 * hf]),
                                          __uint_as_float(y1[4 * q + 2 * hf + 1]));
            const float2 a2 = make_float2(__uint_as_float(y2[4 * q + 2 * hf]),
                                          __uint_as_float(y2[4 * q + 2 * hf + 1]));
            const float2 v = __ffma2_rn(D2, xv, __ffma2_rn(er2, a1, a2));
            *reinterpret_cast<uint32_t*>(yrow + p) = pack_bf16(v.x, v.y);
          }
        }
      }
      if (i == T - 1) {
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
    }
    tc5::fence_proxy_async();
  }

  // ---- outputs of the last token, TMEM release ---------------------------------
  if (sm.err) {
    if (tid == 0) atomicAdd(&g_wide_wait_timeouts, 1u);
  } else if (!ctrl) {
    if (a.hT) {
      float4* dst = reinterpret_cast<float4*>(a.hT + (bh * NS + n_row) * PD + cb);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        dst[j] = make_float4(hs[4 * j], hs[4 * j + 1], hs[4 * j + 2], hs[4 * j + 3]);
    }
    if (a.angleT && tid < NH)
      a.angleT[bh * NH + tid] = ROT ? sm.Phi[tid] : (a.angle0 ? a.angle0[bh * NH + tid] : 0.f);
    if (a.xprevT && tid < PD)
      a.xprevT[bh * PD + tid] = __bfloat162float(Xg[((b * L + L - 1) * H + h) * PD + tid]);
    if (a.bprevT && h % (H / G) == 0 && tid < NS)
      a.bprevT[(b * G + g) * NS + tid] = __bfloat162float(Bg[((b * L + L - 1) * G + g) * NS + tid]);
  }
  tc5::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc5::tmem_dealloc(tmem, kTmemCols);
}

template <int T, bool ROT>
cudaError_t launch_wide(const FwdArgs& a, cudaStream_t s) {
  WMaps tm;
  memset(&tm, 0, sizeof(tm));
  const uint64_t L = (uint64_t)a.L, b = (uint64_t)a.b, H = (uint64_t)a.H, G = (uint64_t)a.G;
  bool ok = encode_map(&tm.B, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.B, NS, G, L, b, 2, 64,
                       CU_TENSOR_MAP_SWIZZLE_128B) &&
            encode_map(&tm.C, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.C, NS, G, L, b, 2, 64,
                       CU_TENSOR_MAP_SWIZZLE_128B) &&
            encode_map(&tm.X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.X, PD, H, L, b, 2, 64,
                       CU_TENSOR_MAP_SWIZZLE_128B);
  if (ok && a.theta)
    ok = encode_map(&tm.theta, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, a.theta, NH, H, L, b, 4, NH,
                    CU_TENSOR_MAP_SWIZZLE_NONE);
  if (!ok) return cudaErrorInvalidValue;
  const size_t smem = sizeof(WSmem<T>) + 1024;
  cudaError_t e = cudaFuncSetAttribute(fwd_chunk_wide_kernel<T, ROT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  fwd_chunk_wide_kernel<T, ROT><<<(unsigned)(a.b * a.H), kThreads, smem, s>>>(a, tm);
  return cudaGetLastError();
}

static_assert(sizeof(WSmem<4>) + 1024 <= 232448, "Q = 256 fits one CTA per SM");

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

bool fwd_chunk_wide_supported(const FwdArgs& a) {
  return a.bf16 && a.N == NS && a.P == PD && a.L > 0 && (a.chunk == 128 || a.chunk == 256) &&
         a.x_tok_stride == 0 && a.theta16 == nullptr && a.Bbias == nullptr && a.Cbias == nullptr &&
         al16(a.X) && al16(a.B) && al16(a.C) && al16(a.Y) && al16(a.theta) && al16(a.h0) &&
         al16(a.hT);
}

cudaError_t launch_fwd_chunk_wide(const FwdArgs& a, cudaStream_t s) {
  if (a.b * a.H == 0) return cudaSuccess;
  const bool rot = a.theta != nullptr || a.angle0 != nullptr;
  if (a.chunk == 128) return rot ? launch_wide<2, true>(a, s) : launch_wide<2, false>(a, s);
  if (a.chunk == 256) return rot ? launch_wide<4, true>(a, s) : launch_wide<4, false>(a, s);
  return cudaErrorInvalidValue;
}

cudaError_t read_and_clear_wide_wait_timeouts(unsigned int* count) {
  const unsigned int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(count, g_wide_wait_timeouts, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_wide_wait_timeouts, &zero, sizeof(unsigned int));
}

}  // namespace m3ssd
