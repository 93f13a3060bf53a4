// Chunked backward of the Mamba-3 SISO scan on the sm_100a tensor cores, for
// bf16 X, B, C, dY with N = 128, P = 64 (one CTA of 512 threads per (b, h)).
//
// The algebra is the chunk adjoint of the fp32 chunked backward (bwd_chunk.cu):
// over a chunk of 64 rows (row 0 the carry-in token), with g = dL/dh_end,
// G = Cbar Bbar^T, E = dY X^T, M = W o G, WE = W o E,
//   dh_prev = exp(cs_63) g + Cbar^T (exp(cs) o dY)
//   dX      = M^T dY + W_end o (Bbar g) + D dY
//   dCbar   = (exp(cs) o dY) h_prev^T + WE Bbar
//   dBbar   = (W_end o X) g^T + WE^T Cbar
// and the mask, decay, rotation and angle gradients, as there.  Every product
// runs as tcgen05 MMAs (kind::f16, bf16 operands, fp32 accumulators in TMEM):
// each fp32 operand is split into a bf16 high part and a bf16 residual, and a
// product takes the part products hi x hi, hi x lo, lo x hi and, where the
// result feeds the suffix sums of dtheta, lo x lo; X and dY are bf16 already and
// enter once.  Operand tiles sit in shared memory in the
// 128-byte-swizzled canonical layout, K-major or MN-major as each product
// needs (the same tile serves both ways).  TMEM columns: G | E (then V | M^T dY)
// | Cbar h_prev | dh_prev | dCbar | dBbar.
//
// Per chunk: stage 1 (G, E; then Cbar h_prev, dh_prev, (W_end o X) g^T,
// (exp(cs) o dY) h_prev^T) starts once the rotated operands are stored; the
// mask gradients read G and E from TMEM and write M and WE; stage 2 (B g,
// M^T dY, WE Bbar, WE^T Cbar) adds onto dCbar and dBbar; the epilogue reads
// everything back for dX, the rotation adjoints, dphi and the carries.  Pass 1
// walks the chunks forward with the state product (W_end o Bbar)^T X on the
// tensor cores and stores each chunk-start state and angle in the workspace.
// The chunk inputs (X, dY, B, C, theta) arrive one chunk ahead by TMA tensor
// copies on a byte-counting mbarrier, straight into the swizzled tiles.
// All cross-thread sums run in a fixed order, so results are deterministic.
// Every mbarrier wait is bounded (2 s) and sets an error flag the host reads.
#include <cuda_bf16.h>

#include <cstring>

#include "common.cuh"
#include "internal.h"
#include "tc5.cuh"

namespace m3ssd {

// Number of bounded device-side waits of this kernel that ran out.
__device__ unsigned int g_bwd_tc_wait_timeouts;

namespace {

constexpr int kQ = 64, QT = kQ - 1, kN = 128, kNH = kN / 2, kP = 64, kT = 512;
constexpr uint32_t kAtom = kQ * 128;  // one 64-element-wide atom of a 64-row bf16 tile
constexpr uint32_t kT1 = kAtom;       // 64 rows x 64 bf16
constexpr uint32_t kT2 = 2 * kAtom;   // 64 rows x 128 bf16
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr uint32_t kColG = 0, kColE = 64, kColY = 128, kColDH = 192, kColDC = 256, kColDB = 384;

typedef __nv_bfloat16 bf16;

// Byte offset of element (r, n) of a 64-row tile of 128-element rows (two
// 64-element atoms of 128-byte rows, 16-byte XOR swizzle).
__device__ __forceinline__ uint32_t off2(int r, int n) {
  return (uint32_t)((n >> 6) * kAtom + r * 128 + ((((n & 63) >> 3) ^ (r & 7)) << 4) +
                    ((n & 7) << 1));
}
// Byte offset of element (r, c) of a tile of 64-element (128-byte) rows.
__device__ __forceinline__ uint32_t off1(int r, int c) {
  return (uint32_t)(r * 128 + ((((c >> 3) ^ (r & 7))) << 4) + ((c & 7) << 1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}
// two fp32 values as a bf16 high pair and a bf16 residual pair
__device__ __forceinline__ void split2(float a, float b, uint32_t& hi, uint32_t& lo) {
  hi = pack_bf16(a, b);
  const float2 h = unpack_bf16(hi);
  lo = pack_bf16(a - h.x, b - h.y);
}
__device__ __forceinline__ float half_sum4(float v) {  // over lanes differing in bits 0-1
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  v += __shfl_xor_sync(0xffffffffu, v, 2);
  return v;
}
__device__ __forceinline__ float col_sum8(float v) {  // over lanes differing in bits 2-4
  v += __shfl_xor_sync(0xffffffffu, v, 4);
  v += __shfl_xor_sync(0xffffffffu, v, 8);
  v += __shfl_xor_sync(0xffffffffu, v, 16);
  return v;
}

// Tensor maps of the chunk inputs: 64-token boxes (token coordinate of row 0
// first; -1 and tokens past the end read as zeros).  X and dY (p, h, t, b), B
// and C (n, g, t, b) in two 64-column boxes, all 128-byte swizzled into the
// operand tiles' layout; theta (i, h, t, b) fp32, unswizzled (r, i) rows.
struct BwdMaps {
  CUtensorMap X, Y, B, C, theta;
};
constexpr uint32_t kBytesX = kT1, kBytesBC = kT2, kBytesTh = kQ * kNH * 4;

struct SmT {
  uint8_t Bh[kT2], Bl[kT2];      // Bbar (u, n)
  uint8_t Ch[kT2], Cl[kT2];      // Cbar (r, n)
  uint8_t Gh[kT2], Gl[kT2];      // g (n, p); in pass 1 W_end o Bbar (u, n)
  uint8_t Hh[kT2], Hl[kT2];      // h_prev (n, p)
  uint8_t X[kT1], Xl[kT1];       // X (u, p); Xl: residual of the cache's fp32 carry-in row
  uint8_t Y[kT1];                // dY (r, p)
  uint8_t EYh[kT1], EYl[kT1];    // exp(cs) o dY (r, p); then M (r, u); then dphi (fp32)
  uint8_t WXh[kT1], WXl[kT1];    // W_end o X (u, p); then WE (r, u)
  float Vt[kQ * kNH];            // theta (r, i), then the angles
  float cs[kQ], al[kQ], ga[kQ], be[kQ], cv[kQ], ecs[kQ], wend[kQ];
  float dcsA[kQ], dcsB[kQ], dcv[kQ], dga[kQ], dwend[kQ], dcsY[kQ];
  float rowp[4][kQ], rowq[4][kQ], rowd[4][kQ];  // per-column-quarter row partials
  float colB[4][kQ], colV[4][kQ];                // per-row-quarter column partials (adjacent)
  float red[kT / 32];
  float phi0[kNH];
  float cdx[2][kP];
  float cdb[2][kN];
  float run[kNH];
  float misc[8];
  uint64_t mbar[3];
  uint64_t lbar;                 // the chunk inputs' TMA copies
  uint32_t tmem;
  uint32_t err;
};
static_assert(sizeof(SmT) + 1024 <= 232448, "one CTA's shared memory");
static_assert(2 * kT1 >= kQ * kNH * 4, "dphi fits in the EY tiles");
static_assert(offsetof(SmT, Hl) == offsetof(SmT, Hh) + kT2, "one bulk copy lands both h_prev tiles");

__device__ __forceinline__ float block_sum(float v, float* red, float* out) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (threadIdx.x == 0) {
    float s = 0.f;
    for (int w = 0; w < kT / 32; ++w) s += red[w];
    *out = s;
  }
  __syncthreads();
  return *out;
}

// Descriptor helpers.  K-major tiles: 128-byte rows along K, 8-row groups 1024 B
// apart; a K step of 16 elements is 32 bytes, and a 128-wide tile moves to its
// second atom after four steps.  MN-major tiles: rows along K, the M or N
// extent along the row in 64-element atoms kAtom apart; a K step is 16 rows.
__device__ __forceinline__ uint64_t dk2(uint32_t a, int j) {
  return tc5::desc_sw128(a, 16, 1024) + (uint64_t)((((j >> 2) * kAtom) + (j & 3) * 32) >> 4);
}
__device__ __forceinline__ uint64_t dk1(uint32_t a, int j) {
  return tc5::desc_sw128(a, 16, 1024) + (uint64_t)((j * 32) >> 4);
}
__device__ __forceinline__ uint64_t dmn(uint32_t a, int j) {
  return tc5::desc_sw128(a, kAtom, 1024) + (uint64_t)((j * 2048) >> 4);
}

constexpr uint32_t kI64 = tc5::idesc_bf16(64, 64, false, false);
constexpr uint32_t kI64mn = tc5::idesc_bf16(64, 64, true, true);
constexpr uint32_t kI128S = tc5::idesc_bf16(128, 64, true, true);
constexpr uint32_t kIN128 = tc5::idesc_bf16(64, 128, false, true);
constexpr uint32_t kIN128k = tc5::idesc_bf16(64, 128, false, false);
constexpr uint32_t kI64kmn = tc5::idesc_bf16(64, 64, false, true);
constexpr uint32_t kIN128mn = tc5::idesc_bf16(64, 128, true, true);

// (hi + lo) x (hi + lo) of a product whose K steps run over `steps`.  `full`
// takes all four part products; otherwise the lo x lo part (at most 2^-16 of a
// product term) is dropped.  Dropping it is a biased error, which the suffix
// sums over later tokens (dtheta) collect: the products that feed dCbar,
// dBbar and dh_prev take it, the others (G, Cbar h_prev, Bbar g) do not.
template <typename FA, typename FB>
__device__ __forceinline__ void mma_split(uint32_t d, uint32_t ah, uint32_t al, uint32_t bh,
                                          uint32_t bl, uint32_t idesc, int steps, bool acc,
                                          bool full, FA da, FB db) {
  for (int j = 0; j < steps; ++j) tc5::mma_bf16(d, da(ah, j), db(bh, j), idesc, acc || j > 0);
  for (int j = 0; j < steps; ++j) tc5::mma_bf16(d, da(ah, j), db(bl, j), idesc, true);
  for (int j = 0; j < steps; ++j) tc5::mma_bf16(d, da(al, j), db(bh, j), idesc, true);
  if (full)
    for (int j = 0; j < steps; ++j) tc5::mma_bf16(d, da(al, j), db(bl, j), idesc, true);
}

__global__ void __launch_bounds__(kT, 1)
    bwd_tc_kernel(BwdArgs a, ChunkWs ws, const __grid_constant__ BwdMaps tm) {
  extern __shared__ uint8_t smraw[];
  SmT& sm = *reinterpret_cast<SmT*>((reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int s4 = warp & 3, q4 = warp >> 2;  // TMEM lane quarter, column quarter
  const uint32_t tl = (uint32_t)(32 * s4) << 16;
  const int ra = 16 * s4 + (lane >> 2), rb = ra + 8;  // rows of an M = 64 result
  const int cq = 2 * (lane & 3);                        // column offset within 8
  const int nrow = 32 * s4 + lane;                      // row of an M = 128 result
  const int64_t H = a.H, G = a.G, L = a.L;
  const int64_t bh = blockIdx.x, b = bh / H, h = bh % H, g = h / (H / G);
  const int nC = (int)((L + QT - 1) / QT);
  const float Dh = a.D ? a.D[h] : 0.f;
  char* wsb = static_cast<char*>(a.workspace);
  // chunk-start states as h_prev tile pairs (bf16 high part, then residual;
  // (n, p), 128-byte swizzled as in shared memory), 2 kT2 bytes a chunk
  uint8_t* hs_img = reinterpret_cast<uint8_t*>(wsb + ws.hs) + bh * (int64_t)nC * (2 * kT2);
  float* ph_ws = reinterpret_cast<float*>(wsb + ws.phs) + bh * (int64_t)nC * kNH;
  float* dBh = reinterpret_cast<float*>(wsb + ws.dBh);
  float* dCh = reinterpret_cast<float*>(wsb + ws.dCh);
  float* dbph = reinterpret_cast<float*>(wsb + ws.dbph);
  float* dDbh = reinterpret_cast<float*>(wsb + ws.dDbh);

  const uint32_t aBh = tc5::saddr(sm.Bh), aBl = tc5::saddr(sm.Bl);
  const uint32_t aCh = tc5::saddr(sm.Ch), aCl = tc5::saddr(sm.Cl);
  const uint32_t aGh = tc5::saddr(sm.Gh), aGl = tc5::saddr(sm.Gl);
  const uint32_t aHh = tc5::saddr(sm.Hh), aHl = tc5::saddr(sm.Hl);
  const uint32_t aX = tc5::saddr(sm.X), aXl = tc5::saddr(sm.Xl), aY = tc5::saddr(sm.Y);
  const uint32_t aEh = tc5::saddr(sm.EYh), aEl = tc5::saddr(sm.EYl);
  const uint32_t aWh = tc5::saddr(sm.WXh), aWl = tc5::saddr(sm.WXl);
  float* dphi = reinterpret_cast<float*>(sm.EYh);  // (r, i), once stage 2 is done
  float* seg = &sm.colB[0][0];                       // 8 x 64 scratch (colB, colV)

  // ---- setup: TMEM, mbarriers, the zero residual rows of X ------------------
  if (warp == 0) tc5::tmem_alloc(&sm.tmem, 512);
  if (tid == 0) {
    for (int k = 0; k < 3; ++k) tc5::mbar_init(&sm.mbar[k], 1);
    tc5::mbar_init(&sm.lbar, 1);
    tc5::fence_mbar_init();
    sm.err = 0;
  }
  for (int e = tid; e < (int)(kT1 / 16); e += kT)
    reinterpret_cast<uint4*>(sm.Xl)[e] = make_uint4(0u, 0u, 0u, 0u);
  if (tid < kNH) sm.phi0[tid] = wrap_angle(a.angle0 ? a.angle0[bh * kNH + tid] : 0.f);
  tc5::fence_before_sync();
  __syncthreads();
  tc5::fence_after_sync();
  const uint32_t tmem = sm.tmem;
  uint32_t par[3] = {0u, 0u, 0u}, lpar = 0u;
  auto wait_bar = [&](int k) {
    if (!tc5::mbar_wait(&sm.mbar[k], par[k], kWaitNs, &sm.err)) sm.err = 1;
    par[k] ^= 1u;
    tc5::fence_after_sync();
  };
  auto wait_loads = [&]() {  // every thread: this chunk's TMA copies have landed
    if (!tc5::mbar_wait(&sm.lbar, lpar, kWaitNs, &sm.err)) sm.err = 1;
    lpar ^= 1u;
  };
  const bool has_th = a.theta != nullptr;
  const int hh = (int)h, gg_ = (int)g, bb = (int)b;
  auto mma_fence_sync = [&]() {  // operand stores -> tensor-core reads
    tc5::fence_proxy_async();
    tc5::fence_before_sync();
    __syncthreads();
    tc5::fence_after_sync();
  };

  // ---- the state pass's inputs, one chunk ahead, by TMA on lbar: theta and raw
  // B rows once the rotation has read the previous ones, X once the state
  // product has (one transaction count covers both); thread (r = tid / 8,
  // sg = tid % 8) then owns X columns 8 sg .., theta pairs 8 sg .. and B columns
  // 16 sg .. of row r
  const int lr = tid >> 3, sg = tid & 7;
  float braw[16], craw[16], xf8[8], yf8[8];
  float sc1[3] = {0.f, 0.f, 0.f};  // logdecay, gamma, beta of row tid (tid < 64)
  auto fetch1_tb = [&](int c) {  // theta, raw B, the scalars
    const int t0 = c * QT - 1;
    if (tid == 0) {
      tc5::mbar_arrive_expect_tx(&sm.lbar, kBytesBC + kBytesX + (has_th ? kBytesTh : 0u));
      if (has_th) tc5::tma_load_4d(tc5::saddr(sm.Vt), &tm.theta, &sm.lbar, 0, hh, t0, bb);
      tc5::tma_load_4d(tc5::saddr(sm.Bh), &tm.B, &sm.lbar, 0, gg_, t0, bb);
      tc5::tma_load_4d(tc5::saddr(sm.Bh) + kAtom, &tm.B, &sm.lbar, 64, gg_, t0, bb);
    }
    sc1[0] = sc1[1] = sc1[2] = 0.f;
    if (tid < kQ && tid > 0 && (int64_t)t0 + tid < L) {
      const int64_t ts = (b * L + t0 + tid) * H + h;
      sc1[0] = a.logdecay[ts];
      sc1[1] = a.gamma[ts];
      sc1[2] = a.beta ? a.beta[ts] : 0.f;
    }
  };
  auto fetch1_x = [&](int c) {
    if (tid == 0) tc5::tma_load_4d(tc5::saddr(sm.X), &tm.X, &sm.lbar, 0, hh, c * QT - 1, bb);
  };
  // theta of row 0 (the carry-in token's own angle step belongs to the chunk
  // before) is zero; so is all of theta when there is none
  auto zero_theta = [&]() {
    if (lr == 0 || !has_th) {
      *reinterpret_cast<float4*>(&sm.Vt[lr * kNH + 8 * sg]) = make_float4(0.f, 0.f, 0.f, 0.f);
      *reinterpret_cast<float4*>(&sm.Vt[lr * kNH + 8 * sg + 4]) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  auto commit1 = [&](int c) {
    wait_loads();
    zero_theta();
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float2 fb = unpack_bf16(*reinterpret_cast<const uint32_t*>(sm.Bh + off2(lr, 16 * sg + 2 * q)));
      braw[2 * q] = fb.x;
      braw[2 * q + 1] = fb.y;
    }
    if ((int64_t)c * QT - 1 + lr == -1) {  // the cache's carry-in token, fp32
      float xf[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) xf[k] = a.xprev0 ? a.xprev0[bh * kP + 8 * sg + k] : 0.f;
#pragma unroll
      for (int k = 0; k < 16; ++k) braw[k] = a.bprev0 ? a.bprev0[(b * G + g) * kN + 16 * sg + k] : 0.f;
      uint32_t hi[4], lo[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) split2(xf[2 * q], xf[2 * q + 1], hi[q], lo[q]);
      *reinterpret_cast<uint4*>(sm.X + off1(0, 8 * sg)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<uint4*>(sm.Xl + off1(0, 8 * sg)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
    if (tid < kQ) {
      sm.cs[tid] = sc1[0];  // the raw logdecay until scalars_angles
      sm.ga[tid] = sc1[1];
      sm.be[tid] = sc1[2];
    }
  };

  // ---- chunk scalars (cs, alpha, exp(cs), cv, W_end: warp 0 alone, rows lane and
  // lane + 32, neighbours by shuffle) and the angles phi(r, i) = phi0[i] +
  // sum_{k <= r} theta(k, i) (all threads, in 8-row segments); two barriers
  auto scalars_angles = [&]() {
    if (warp == 0) {
      const float l0 = sm.cs[lane], l1 = sm.cs[lane + 32];  // raw logdecay
      const float g0 = sm.ga[lane], g1 = sm.ga[lane + 32];
      const float e0 = sm.be[lane], e1 = sm.be[lane + 32];
      float s0 = l0, s1 = l1;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float v0 = __shfl_up_sync(0xffffffffu, s0, o);
        const float v1 = __shfl_up_sync(0xffffffffu, s1, o);
        if (lane >= o) {
          s0 += v0;
          s1 += v1;
        }
      }
      s1 += __shfl_sync(0xffffffffu, s0, 31);
      const float a0 = expf(l0), a1 = expf(l1);
      // the row after: lane + 1 (row 32 for lane 31), lane + 33
      const float a0n = __shfl_down_sync(0xffffffffu, a0, 1), a1n = __shfl_down_sync(0xffffffffu, a1, 1);
      const float e0n = __shfl_down_sync(0xffffffffu, e0, 1), e1n = __shfl_down_sync(0xffffffffu, e1, 1);
      const float s0n = __shfl_down_sync(0xffffffffu, s0, 1), s1n = __shfl_down_sync(0xffffffffu, s1, 1);
      const float a32 = __shfl_sync(0xffffffffu, a1, 0), e32 = __shfl_sync(0xffffffffu, e1, 0);
      const float s32 = __shfl_sync(0xffffffffu, s1, 0), s63 = __shfl_sync(0xffffffffu, s1, 31);
      const bool last = lane == 31;
      const float cv0 = g0 * (last ? a32 : a0n) + (last ? e32 : e0n);
      const float cv1 = last ? 0.f : g1 * a1n + e1n;
      sm.cs[lane] = s0;
      sm.cs[lane + 32] = s1;
      sm.al[lane] = a0;
      sm.al[lane + 32] = a1;
      sm.ecs[lane] = expf(s0);
      sm.ecs[lane + 32] = expf(s1);
      sm.cv[lane] = cv0;
      sm.cv[lane + 32] = cv1;
      sm.wend[lane] = expf(s63 - (last ? s32 : s0n)) * cv0;
      sm.wend[lane + 32] = last ? g1 : expf(s63 - s1n) * cv1;
    }
    const int i = tid & 63, grp = tid >> 6;
    float run_ = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int r = 8 * grp + k;
      run_ += sm.Vt[r * kNH + i];
      sm.Vt[r * kNH + i] = run_;
    }
    seg[grp * kNH + i] = run_;  // segment totals
    __syncthreads();
    float base = sm.phi0[i];
    for (int q = 0; q < grp; ++q) base += seg[q * kNH + i];
#pragma unroll
    for (int k = 0; k < 8; ++k) sm.Vt[(8 * grp + k) * kNH + i] += base;
    __syncthreads();
  };

  // ---- rotation of this thread's row segment (pairs 8 sg .. 8 sg + 7) ---------
  // pass 1: W_end(r) Bbar_r into the g tiles; pass 2: Bbar and Cbar, then the
  // tiles exp(cs) o dY and W_end o X
  auto st32 = [](uint8_t* base, uint32_t off, uint32_t v) {
    *reinterpret_cast<uint32_t*>(base + off) = v;
  };
  auto st128 = [](uint8_t* base, uint32_t off, const uint32_t* v) {
    *reinterpret_cast<uint4*>(base + off) = make_uint4(v[0], v[1], v[2], v[3]);
  };
  auto rotate = [&](bool bwd) {
    const int r = lr;
    const float we = sm.wend[r];
    uint32_t bh_[8], bl_[8], ch_[8], cl_[8];  // 16 columns 16 sg .. as bf16 pairs
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int i = 8 * sg + k;
      float sn, cs_;
      fast_sincos(sm.Vt[r * kNH + i], &sn, &cs_);
      const float b0 = braw[2 * k], b1 = braw[2 * k + 1];
      const float bb0 = cs_ * b0 - sn * b1, bb1 = sn * b0 + cs_ * b1;
      if (!bwd) {
        split2(we * bb0, we * bb1, bh_[k], bl_[k]);
      } else {
        split2(bb0, bb1, bh_[k], bl_[k]);
        const float c0 = craw[2 * k], c1 = craw[2 * k + 1];
        split2(cs_ * c0 - sn * c1, sn * c0 + cs_ * c1, ch_[k], cl_[k]);
      }
    }
    uint8_t* th_ = bwd ? sm.Bh : sm.Gh;
    uint8_t* tl_ = bwd ? sm.Bl : sm.Gl;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const uint32_t o = off2(r, 16 * sg + 8 * half);  // a 16-byte chunk of 8 columns
      st128(th_, o, bh_ + 4 * half);
      st128(tl_, o, bl_ + 4 * half);
      if (bwd) {
        st128(sm.Ch, o, ch_ + 4 * half);
        st128(sm.Cl, o, cl_ + 4 * half);
      }
    }
    if (bwd) {
      const float e = sm.ecs[r];
      uint32_t eh[4], el[4], xh[4], xl[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        split2(e * yf8[2 * q], e * yf8[2 * q + 1], eh[q], el[q]);
        split2(we * xf8[2 * q], we * xf8[2 * q + 1], xh[q], xl[q]);
      }
      const uint32_t o = off1(r, 8 * sg);
      st128(sm.EYh, o, eh);
      st128(sm.EYl, o, el);
      st128(sm.WXh, o, xh);
      st128(sm.WXl, o, xl);
    }
  };
  // an (n, p) tile pair from the thread's 16 values (row nrow, columns 16 q4 ..)
  auto store_np = [&](uint8_t* hi_t, uint8_t* lo_t, const float* v) {
    uint32_t hv[8], lv[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) split2(v[2 * q], v[2 * q + 1], hv[q], lv[q]);
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const uint32_t o = off1(nrow, 16 * q4 + 8 * half);
      st128(hi_t, o, hv + 4 * half);
      st128(lo_t, o, lv + 4 * half);
    }
  };

  // ---- the reverse pass's inputs one chunk ahead: the chunk-start state's
  // tiles by a bulk copy (fetch_h, once stage 1 has read the previous ones); X,
  // dY, theta and raw B, C rows by TMA into their tiles (free from the end of
  // the previous chunk's epilogue on); the scalars and the chunk-start angle
  // into registers; commit_chunk() lands them
  struct Pre {
    float sc[3];
    float ph;
  };
  // the chunk-start state's tile pair, one bulk copy, as soon as the previous
  // chunk's products have read its own (stage 1); it opens the loads' phase for
  // all of the chunk's copies
  auto fetch_h = [&](int c) {
    if (tid == 0) {
      tc5::mbar_arrive_expect_tx(&sm.lbar, 2 * kT2 + 2 * kBytesX + 2 * kBytesBC + (has_th ? kBytesTh : 0u));
      tc5::bulk_load(tc5::saddr(sm.Hh), hs_img + (int64_t)c * (2 * kT2), 2 * kT2, &sm.lbar);
    }
  };
  auto fetch_chunk = [&](int c, Pre& f) {
    const int64_t t0 = (int64_t)c * QT - 1;
    if (tid == 0) {
      const int tc = (int)t0;
      const uint32_t aB = tc5::saddr(sm.Bh), aC = tc5::saddr(sm.Ch);
      tc5::tma_load_4d(tc5::saddr(sm.X), &tm.X, &sm.lbar, 0, hh, tc, bb);
      tc5::tma_load_4d(tc5::saddr(sm.Y), &tm.Y, &sm.lbar, 0, hh, tc, bb);
      tc5::tma_load_4d(aB, &tm.B, &sm.lbar, 0, gg_, tc, bb);
      tc5::tma_load_4d(aB + kAtom, &tm.B, &sm.lbar, 64, gg_, tc, bb);
      tc5::tma_load_4d(aC, &tm.C, &sm.lbar, 0, gg_, tc, bb);
      tc5::tma_load_4d(aC + kAtom, &tm.C, &sm.lbar, 64, gg_, tc, bb);
      if (has_th) tc5::tma_load_4d(tc5::saddr(sm.Vt), &tm.theta, &sm.lbar, 0, hh, tc, bb);
    }
    f.sc[0] = f.sc[1] = f.sc[2] = 0.f;
    f.ph = 0.f;
    if (tid < kQ) {
      if (tid > 0 && t0 + tid < L) {
        const int64_t ts = (b * L + t0 + tid) * H + h;
        f.sc[0] = a.logdecay[ts];
        f.sc[1] = a.gamma[ts];
        f.sc[2] = a.beta ? a.beta[ts] : 0.f;
      }
      if (tid < kNH) f.ph = ph_ws[(int64_t)c * kNH + tid];
    }
  };
  auto commit_chunk = [&](int c, const Pre& f) {
    wait_loads();
    const int64_t t0 = (int64_t)c * QT - 1;
    // row 0 is the carry-in token: its dY and C belong to the chunk before
    zero_theta();
    if (lr == 0) {
      const uint4 z = make_uint4(0u, 0u, 0u, 0u);
      *reinterpret_cast<uint4*>(sm.Y + off1(0, 8 * sg)) = z;
      *reinterpret_cast<uint4*>(sm.Ch + off2(0, 16 * sg)) = z;
      *reinterpret_cast<uint4*>(sm.Ch + off2(0, 16 * sg + 8)) = z;
    }
    // this thread's raw B, C (16 columns) and x, dy (8 columns) in fp32
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int n = 16 * sg + 2 * q;
      const float2 fb = unpack_bf16(*reinterpret_cast<const uint32_t*>(sm.Bh + off2(lr, n)));
      const float2 fc = unpack_bf16(*reinterpret_cast<const uint32_t*>(sm.Ch + off2(lr, n)));
      braw[2 * q] = fb.x;
      braw[2 * q + 1] = fb.y;
      craw[2 * q] = fc.x;
      craw[2 * q + 1] = fc.y;
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int p = 8 * sg + 2 * q;
      const float2 fx = unpack_bf16(*reinterpret_cast<const uint32_t*>(sm.X + off1(lr, p)));
      const float2 fy = unpack_bf16(*reinterpret_cast<const uint32_t*>(sm.Y + off1(lr, p)));
      xf8[2 * q] = fx.x;
      xf8[2 * q + 1] = fx.y;
      yf8[2 * q] = fy.x;
      yf8[2 * q + 1] = fy.y;
    }
    if (t0 + lr == -1) {  // the cache's carry-in token, fp32
#pragma unroll
      for (int k = 0; k < 8; ++k) xf8[k] = a.xprev0 ? a.xprev0[bh * kP + 8 * sg + k] : 0.f;
#pragma unroll
      for (int k = 0; k < 16; ++k) braw[k] = a.bprev0 ? a.bprev0[(b * G + g) * kN + 16 * sg + k] : 0.f;
      uint32_t hi[4], lo[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) split2(xf8[2 * q], xf8[2 * q + 1], hi[q], lo[q]);
      *reinterpret_cast<uint4*>(sm.X + off1(0, 8 * sg)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<uint4*>(sm.Xl + off1(0, 8 * sg)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
    if (tid < kQ) {
      sm.cs[tid] = f.sc[0];  // the raw logdecay until scalars_angles
      sm.ga[tid] = f.sc[1];
      sm.be[tid] = f.sc[2];
      if (tid < kNH) sm.phi0[tid] = f.ph;
    }
  };

  const auto K2 = [](uint32_t ad, int j) { return dk2(ad, j); };
  const auto K1 = [](uint32_t ad, int j) { return dk1(ad, j); };
  const auto MN = [](uint32_t ad, int j) { return dmn(ad, j); };
  const bool has_xl = a.xprev0 != nullptr;

  // ---- pass 1: the state and the angle at every chunk start -----------------
  float hreg[16];  // h rows nrow, columns 16 q4 + j
#pragma unroll
  for (int j = 0; j < 16; ++j) hreg[j] = a.h0 ? a.h0[(bh * kN + nrow) * kP + 16 * q4 + j] : 0.f;
  if (nC > 0) {
    fetch1_tb(0);
    fetch1_x(0);
  }
  for (int c = 0; c < nC; ++c) {
    store_np(hs_img + (int64_t)c * (2 * kT2), hs_img + (int64_t)c * (2 * kT2) + kT2, hreg);
    if (tid < kNH) ph_ws[(int64_t)c * kNH + tid] = sm.phi0[tid];
    commit1(c);
    __syncthreads();
    scalars_angles();
    const float nphi = tid < kNH ? wrap_angle(sm.Vt[(kQ - 1) * kNH + tid]) : 0.f;
    rotate(false);
    mma_fence_sync();  // the rotation has read theta and B: the next ones may land
    if (c + 1 < nC) fetch1_tb(c + 1);
    if (tid == 0) {
      // S = (W_end o Bbar)^T X: A MN-major (M = n), B MN-major (N = p), K = u
      for (int j = 0; j < 4; ++j) tc5::mma_bf16(tmem + kColG, dmn(aGh, j), dmn(aX, j), kI128S, j > 0);
      for (int j = 0; j < 4; ++j) tc5::mma_bf16(tmem + kColG, dmn(aGl, j), dmn(aX, j), kI128S, true);
      if (c == 0 && has_xl)
        for (int j = 0; j < 4; ++j) tc5::mma_bf16(tmem + kColG, dmn(aGh, j), dmn(aXl, j), kI128S, true);
      tc5::commit(&sm.mbar[0]);
    }
    wait_bar(0);
    if (c + 1 < nC) fetch1_x(c + 1);  // the state product has read X
    uint32_t sv[16];
    tc5::ld_32x32b_x16(tmem + tl + kColG + (uint32_t)(16 * q4), sv);
    tc5::wait_ld();
    const float eE = sm.ecs[kQ - 1];
#pragma unroll
    for (int j = 0; j < 16; ++j) hreg[j] = fmaf(eE, hreg[j], __uint_as_float(sv[j]));
    tc5::fence_before_sync();
    __syncthreads();  // every read of this chunk's scalars and columns is done
    tc5::fence_after_sync();
    if (tid < kNH) sm.phi0[tid] = nphi;
  }

  tc5::fence_proxy_async_global();  // the state images -> the bulk copies below
  __syncthreads();

  // ---- pass 2: the chunks in reverse --------------------------------------
  float greg[16];  // g = dL/dh_end, rows nrow, columns 16 q4 + j
#pragma unroll
  for (int j = 0; j < 16; ++j) greg[j] = a.dhT ? a.dhT[(bh * kN + nrow) * kP + 16 * q4 + j] : 0.f;
  store_np(sm.Gh, sm.Gl, greg);
  if (tid < kNH) sm.run[tid] = 0.f;
  if (tid < kP) sm.cdx[0][tid] = sm.cdx[1][tid] = 0.f;
  if (tid < kN) sm.cdb[0][tid] = sm.cdb[1][tid] = 0.f;
  float dDacc = 0.f;
  Pre f;
  if (nC > 0) {
    fetch_h(nC - 1);
    fetch_chunk(nC - 1, f);
  }
  __syncthreads();

  for (int c = nC - 1; c >= 0; --c) {
    const int cur = c & 1, nxt = cur ^ 1;
    const int64_t t0 = (int64_t)c * QT - 1;
    auto own = [&](int r) { return r > 0 && t0 + r < L; };
    commit_chunk(c, f);
    __syncthreads();
    scalars_angles();
    rotate(true);
    mma_fence_sync();

    // -- stage 1
    if (tid == 0) {
      mma_split(tmem + kColG, aCh, aCl, aBh, aBl, kI64, 8, false, false, K2, K2);  // G
      for (int j = 0; j < 4; ++j) tc5::mma_bf16(tmem + kColE, dk1(aY, j), dk1(aX, j), kI64, j > 0);
      if (c == 0 && has_xl)
        for (int j = 0; j < 4; ++j) tc5::mma_bf16(tmem + kColE, dk1(aY, j), dk1(aXl, j), kI64, true);
      tc5::commit(&sm.mbar[0]);                                          // G, E
      mma_split(tmem + kColY, aCh, aCl, aHh, aHl, kI64kmn, 8, false, false, K2, MN);  // Cbar h_prev
      mma_split(tmem + kColDH, aCh, aCl, aEh, aEl, kI128S, 4, false, true, MN, MN); // Cbar^T e^cs dY
      mma_split(tmem + kColDB, aWh, aWl, aGh, aGl, kIN128k, 4, false, true, K1, K1); // (W_end X) g^T
      mma_split(tmem + kColDC, aEh, aEl, aHh, aHl, kIN128k, 4, false, true, K1, K1); // e^cs dY h_prev^T
      tc5::commit(&sm.mbar[1]);
    }

    // -- the mask gradients from G and E (rows ra, rb; columns 16 q4 + 8 gg + cq + e)
    {
      float wv[2][2][2], xv[2][2][2];
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int r = hf ? rb : ra;
        const float csr = sm.cs[r];
#pragma unroll
        for (int gg = 0; gg < 2; ++gg)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int u = 16 * q4 + 8 * gg + cq + e;
            float w = 0.f, ex = 0.f;
            if (u < r) {
              ex = expf(csr - sm.cs[u + 1]);
              w = ex * sm.cv[u];
            } else if (u == r) {
              w = sm.ga[r];
            }
            wv[hf][gg][e] = w;
            xv[hf][gg][e] = ex;
          }
      }
      wait_bar(0);
      uint32_t gr[8], er[8];
      tc5::ld_16x256b_x2(tmem + tl + kColG + (uint32_t)(16 * q4), gr);
      tc5::ld_16x256b_x2(tmem + tl + kColE + (uint32_t)(16 * q4), er);
      tc5::wait_ld();
      float rowA[2] = {0.f, 0.f}, cB[2][2] = {{0.f, 0.f}, {0.f, 0.f}}, cV[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
      uint32_t mh[2][2], ml[2][2], eh[2][2], el[2][2];
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int r = hf ? rb : ra;
#pragma unroll
        for (int gg = 0; gg < 2; ++gg) {
          float mv[2], wev[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int u = 16 * q4 + 8 * gg + cq + e;
            const float Gv = __uint_as_float(gr[4 * gg + 2 * hf + e]);
            const float Ev = __uint_as_float(er[4 * gg + 2 * hf + e]);
            const float dW = Gv * Ev, w = wv[hf][gg][e];
            if (u < r) {
              rowA[hf] = fmaf(dW, w, rowA[hf]);
              cB[gg][e] = fmaf(dW, w, cB[gg][e]);
              cV[gg][e] = fmaf(dW, xv[hf][gg][e], cV[gg][e]);
            } else if (u == r) {
              sm.dga[r] = dW;
            }
            mv[e] = w * Gv;
            wev[e] = w * Ev;
          }
          split2(mv[0], mv[1], mh[hf][gg], ml[hf][gg]);
          split2(wev[0], wev[1], eh[hf][gg], el[hf][gg]);
        }
      }
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const float v = half_sum4(rowA[hf]);
        if ((lane & 3) == 0) sm.rowp[q4][hf ? rb : ra] = v;
      }
#pragma unroll
      for (int gg = 0; gg < 2; ++gg)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float vb = col_sum8(cB[gg][e]), vv = col_sum8(cV[gg][e]);
          if (lane < 4) {
            const int u = 16 * q4 + 8 * gg + cq + e;
            sm.colB[s4][u] = vb;
            sm.colV[s4][u] = vv;
          }
        }
      wait_bar(1);  // stage 1 done: the e^cs dY and W_end X tiles take M and WE
#pragma unroll
      for (int hf = 0; hf < 2; ++hf)
#pragma unroll
        for (int gg = 0; gg < 2; ++gg) {
          const int r = hf ? rb : ra, u0 = 16 * q4 + 8 * gg + cq;
          st32(sm.EYh, off1(r, u0), mh[hf][gg]);
          st32(sm.EYl, off1(r, u0), ml[hf][gg]);
          st32(sm.WXh, off1(r, u0), eh[hf][gg]);
          st32(sm.WXl, off1(r, u0), el[hf][gg]);
        }
    }

    // -- Cbar h_prev: the h_prev term of d cs_r; dh_prev: the next g
    float ghp = 0.f;
    {
      uint32_t yr[8], dhr[16];
      tc5::ld_16x256b_x2(tmem + tl + kColY + (uint32_t)(16 * q4), yr);
      tc5::ld_32x32b_x16(tmem + tl + kColDH + (uint32_t)(16 * q4), dhr);
      tc5::wait_ld();
      float sy[2] = {0.f, 0.f};
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int r = hf ? rb : ra;
#pragma unroll
        for (int gg = 0; gg < 2; ++gg) {
          const int p0 = 16 * q4 + 8 * gg + cq;
          const float2 dy = unpack_bf16(*reinterpret_cast<const uint32_t*>(sm.Y + off1(r, p0)));
          sy[hf] = fmaf(dy.x, __uint_as_float(yr[4 * gg + 2 * hf]),
                        fmaf(dy.y, __uint_as_float(yr[4 * gg + 2 * hf + 1]), sy[hf]));
        }
        const float v = half_sum4(sy[hf]) * sm.ecs[r];
        if ((lane & 3) == 0) sm.rowq[q4][r] = v;
      }
      float hpr[16];  // h_prev row nrow, columns 16 q4 + j, as its high part + residual
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const uint32_t o = off1(nrow, 16 * q4 + 8 * half);
        const uint4 vh = *reinterpret_cast<const uint4*>(sm.Hh + o);
        const uint4 vl = *reinterpret_cast<const uint4*>(sm.Hl + o);
        const uint32_t uh[4] = {vh.x, vh.y, vh.z, vh.w}, ul[4] = {vl.x, vl.y, vl.z, vl.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 fh = unpack_bf16(uh[q]), fl = unpack_bf16(ul[q]);
          hpr[8 * half + 2 * q] = fh.x + fl.x;
          hpr[8 * half + 2 * q + 1] = fh.y + fl.y;
        }
      }
      const float eE = sm.ecs[kQ - 1];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        ghp = fmaf(greg[j], hpr[j], ghp);
        greg[j] = fmaf(eE, greg[j], __uint_as_float(dhr[j]));
      }
    }
    mma_fence_sync();  // M and WE stored; G, E and h_prev read
    if (c > 0) fetch_h(c - 1);

    // -- stage 2
    if (tid == 0) {
      mma_split(tmem + kColG, aBh, aBl, aGh, aGl, kI64kmn, 8, false, false, K2, MN);  // Bbar g
      for (int j = 0; j < 4; ++j) tc5::mma_bf16(tmem + kColE, dmn(aEh, j), dmn(aY, j), kI64mn, j > 0);
      for (int j = 0; j < 4; ++j) tc5::mma_bf16(tmem + kColE, dmn(aEl, j), dmn(aY, j), kI64mn, true);
      mma_split(tmem + kColDC, aWh, aWl, aBh, aBl, kIN128, 4, true, true, K1, MN);    // += WE Bbar
      mma_split(tmem + kColDB, aWh, aWl, aCh, aCl, kIN128mn, 4, true, true, MN, MN);  // += WE^T Cbar
      tc5::commit(&sm.mbar[2]);
    }
    block_sum(ghp, sm.red, &sm.misc[0]);
    wait_bar(2);

    // -- dX = M^T dY + W_end o (Bbar g) + D dY; dW_end(u) = x_u . (Bbar_u g)
    {
      uint32_t vr[8], mr[8];
      tc5::ld_16x256b_x2(tmem + tl + kColG + (uint32_t)(16 * q4), vr);
      tc5::ld_16x256b_x2(tmem + tl + kColE + (uint32_t)(16 * q4), mr);
      tc5::wait_ld();
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int u = hf ? rb : ra;
        const float we = sm.wend[u];
        float dwe = 0.f;
#pragma unroll
        for (int gg = 0; gg < 2; ++gg) {
          const int p0 = 16 * q4 + 8 * gg + cq;
          const float2 xh = unpack_bf16(*reinterpret_cast<const uint32_t*>(sm.X + off1(u, p0)));
          const float2 xl = c == 0 ? unpack_bf16(*reinterpret_cast<const uint32_t*>(sm.Xl + off1(u, p0)))
                                   : make_float2(0.f, 0.f);  // the carry-in residual: chunk 0 only
          const float2 dy = unpack_bf16(*reinterpret_cast<const uint32_t*>(sm.Y + off1(u, p0)));
          const float xs[2] = {xh.x + xl.x, xh.y + xl.y}, ys[2] = {dy.x, dy.y};
          float dx[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float V = __uint_as_float(vr[4 * gg + 2 * hf + e]);
            dwe = fmaf(xs[e], V, dwe);
            dDacc = fmaf(ys[e], xs[e], dDacc);
            dx[e] = __uint_as_float(mr[4 * gg + 2 * hf + e]) + fmaf(we, V, Dh * ys[e]);
            if (u == kQ - 1) dx[e] += sm.cdx[nxt][p0 + e];
          }
          if (u == 0) {
            sm.cdx[cur][p0] = dx[0];
            sm.cdx[cur][p0 + 1] = dx[1];
          } else if (own(u)) {
            *reinterpret_cast<float2*>(&a.dX[((b * L + t0 + u) * H + h) * kP + p0]) =
                make_float2(dx[0], dx[1]);
          }
        }
        dwe = half_sum4(dwe);
        if ((lane & 3) == 0) sm.rowd[q4][u] = dwe;
      }
    }

    // -- dCbar, dBbar: carries, rotation adjoints, dphi (rows ra, rb; columns
    //    32 q4 + 8 gg + cq + e)
    {
      uint32_t cr[16], br[16];
      tc5::ld_16x256b_x4(tmem + tl + kColDC + (uint32_t)(32 * q4), cr);
      tc5::ld_16x256b_x4(tmem + tl + kColDB + (uint32_t)(32 * q4), br);
      tc5::wait_ld();
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int r = hf ? rb : ra;
        const bool ok = own(r);
        const int64_t ro = ((b * L + (ok ? t0 + r : 0)) * H + h) * kN;
#pragma unroll
        for (int gg = 0; gg < 4; ++gg) {
          const int n = 32 * q4 + 8 * gg + cq, i = n >> 1;
          const float dc0 = __uint_as_float(cr[4 * gg + 2 * hf]);
          const float dc1 = __uint_as_float(cr[4 * gg + 2 * hf + 1]);
          float db0 = __uint_as_float(br[4 * gg + 2 * hf]);
          float db1 = __uint_as_float(br[4 * gg + 2 * hf + 1]);
          if (r == kQ - 1) {
            db0 += sm.cdb[nxt][n];
            db1 += sm.cdb[nxt][n + 1];
          }
          if (r == 0) {
            sm.cdb[cur][n] = db0;
            sm.cdb[cur][n + 1] = db1;
          }
          float dp = 0.f;
          if (ok) {
            float sn, cs_;
            fast_sincos(sm.Vt[r * kNH + i], &sn, &cs_);
            const float2 ch = unpack_bf16(*reinterpret_cast<const uint32_t*>(sm.Ch + off2(r, n)));
            const float2 cl = unpack_bf16(*reinterpret_cast<const uint32_t*>(sm.Cl + off2(r, n)));
            const float2 bh_ = unpack_bf16(*reinterpret_cast<const uint32_t*>(sm.Bh + off2(r, n)));
            const float2 bl_ = unpack_bf16(*reinterpret_cast<const uint32_t*>(sm.Bl + off2(r, n)));
            const float c0 = ch.x + cl.x, c1 = ch.y + cl.y, b0 = bh_.x + bl_.x, b1 = bh_.y + bl_.y;
            dp = fmaf(dc1, c0, -dc0 * c1) + fmaf(db1, b0, -db0 * b1);
            *reinterpret_cast<float2*>(&dCh[ro + n]) =
                make_float2(fmaf(cs_, dc0, sn * dc1), fmaf(cs_, dc1, -sn * dc0));
            *reinterpret_cast<float2*>(&dBh[ro + n]) =
                make_float2(fmaf(cs_, db0, sn * db1), fmaf(cs_, db1, -sn * db0));
          }
          dphi[r * kNH + i] = dp;
        }
      }
    }
    tc5::fence_before_sync();
    __syncthreads();  // the tiles of X, dY, theta and B, C are read: fetch the next chunk
    tc5::fence_after_sync();
    if (c > 0) fetch_chunk(c - 1, f);
    store_np(sm.Gh, sm.Gl, greg);  // the next (earlier) chunk's g
    __syncthreads();

    // -- the scalar chain: decay sums -> cv -> gamma, beta, logdecay (warp 0)
    if (warp == 0) {
      const float eE = sm.ecs[kQ - 1];
      float dw[2], dcsv[2];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int u = lane + 32 * k;
        dw[k] = sm.rowd[0][u] + sm.rowd[1][u] + sm.rowd[2][u] + sm.rowd[3][u];
        sm.dwend[u] = dw[k];
      }
      float endsum = 0.f;
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int u = lane + 32 * k;
        if (u < kQ - 1) endsum = fmaf(dw[k], sm.wend[u], endsum);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) endsum += __shfl_xor_sync(0xffffffffu, endsum, o);
      __syncwarp();
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int r = lane + 32 * k;
        const float dA = sm.rowp[0][r] + sm.rowp[1][r] + sm.rowp[2][r] + sm.rowp[3][r];
        const float dY_ = sm.rowq[0][r] + sm.rowq[1][r] + sm.rowq[2][r] + sm.rowq[3][r];
        float d = dA + dY_;
        if (r >= 1) {
          const int u = r - 1;
          const float dB_ = sm.colB[0][u] + sm.colB[1][u] + sm.colB[2][u] + sm.colB[3][u];
          d -= dB_ + sm.dwend[u] * sm.wend[u];
        }
        if (r == kQ - 1) d += endsum + eE * sm.misc[0];
        dcsv[k] = d;
        float dv = sm.colV[0][r] + sm.colV[1][r] + sm.colV[2][r] + sm.colV[3][r];
        if (r < kQ - 1) dv = fmaf(sm.dwend[r], expf(sm.cs[kQ - 1] - sm.cs[r + 1]), dv);
        sm.dcv[r] = dv;
      }
      __syncwarp();
      float s1 = dcsv[1], s0 = dcsv[0];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float v1 = __shfl_down_sync(0xffffffffu, s1, o);
        const float v0 = __shfl_down_sync(0xffffffffu, s0, o);
        if (lane + o < 32) {
          s1 += v1;
          s0 += v0;
        }
      }
      s0 += __shfl_sync(0xffffffffu, s1, 0);
      const float suf[2] = {s0, s1};
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int r = lane + 32 * k;
        if (!own(r)) continue;
        const float dcvp = sm.dcv[r - 1];
        float dg = sm.dga[r];
        if (r == kQ - 1) dg += sm.dwend[kQ - 1];
        if (r < kQ - 1) dg = fmaf(sm.dcv[r], sm.al[r + 1], dg);
        const float dal = dcvp * sm.ga[r - 1];
        const int64_t th = (b * L + t0 + r) * H + h;
        a.dlogdecay[th] = fmaf(sm.al[r], dal, suf[k]);
        a.dgamma[th] = dg;
        if (a.dbeta) a.dbeta[th] = dcvp;
      }
    }

    // -- dtheta: suffix sums of dphi over the tokens after, in 8-row segments
    {
      float* segd = reinterpret_cast<float*>(sm.WXh);  // WE is dead
      const int i = tid & 63, grp = tid >> 6;
      float tmp[8];
      float sacc = 0.f;
#pragma unroll
      for (int k = 7; k >= 0; --k) {
        sacc += dphi[(8 * grp + k) * kNH + i];
        tmp[k] = sacc;
      }
      segd[grp * kNH + i] = sacc;
      __syncthreads();
      float base = sm.run[i];
      for (int q = 7; q > grp; --q) base += segd[q * kNH + i];
      if (a.dtheta) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int r = 8 * grp + k;
          if (own(r)) a.dtheta[((b * L + t0 + r) * H + h) * kNH + i] = base + tmp[k];
        }
      }
      __syncthreads();
      if (grp == 0) sm.run[i] = base + tmp[0];
      __syncthreads();
    }
  }

  // ---- the cache token before the sequence: dh0, dxprev0, dbprev0, dangle0, dD
  if (a.dh0) {
#pragma unroll
    for (int j = 0; j < 16; ++j) a.dh0[(bh * kN + nrow) * kP + 16 * q4 + j] = greg[j];
  }
  if (a.dxprev0 && tid < kP) a.dxprev0[bh * kP + tid] = sm.cdx[0][tid];
  if (tid < kNH) {
    const int i = tid;
    float sn, cs_;
    fast_sincos(sm.phi0[i], &sn, &cs_);
    const float d0 = sm.cdb[0][2 * i], d1 = sm.cdb[0][2 * i + 1];
    float v0 = 0.f, v1 = 0.f;
    if (a.bprev0) {
      v0 = a.bprev0[(b * G + g) * kN + 2 * i];
      v1 = a.bprev0[(b * G + g) * kN + 2 * i + 1];
    }
    const float vb0 = cs_ * v0 - sn * v1, vb1 = sn * v0 + cs_ * v1;
    dbph[bh * kN + 2 * i] = fmaf(cs_, d0, sn * d1);
    dbph[bh * kN + 2 * i + 1] = fmaf(cs_, d1, -sn * d0);
    if (a.dangle0) a.dangle0[bh * kNH + i] = sm.run[i] + fmaf(d1, vb0, -d0 * vb1);
  }
  const float dDs = block_sum(dDacc, sm.red, &sm.misc[1]);
  if (tid == 0) {
    dDbh[bh] = dDs;
    if (sm.err) {
      atomicAdd(&g_bwd_tc_wait_timeouts, 1u);
      // a wait gave up: let the last copies and products in flight land (each
      // wait again bounded) before the CTA's shared memory and TMEM go
      tc5::mbar_wait(&sm.lbar, lpar ^ 1u, kWaitNs);
      for (int k = 0; k < 3; ++k) tc5::mbar_wait(&sm.mbar[k], par[k] ^ 1u, kWaitNs);
    }
  }
  tc5::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc5::tmem_dealloc(tmem, 512);
}

}  // namespace

bool bwd_tc_supported(const BwdArgs& a) {
  auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
  return a.bf16 && a.N == kN && a.P == kP && al16(a.X) && al16(a.B) && al16(a.C) &&
         al16(a.dY) && al16(a.theta);
}

cudaError_t launch_bwd_tc(const BwdArgs& a, cudaStream_t s) {
  if (a.b * a.H == 0) return cudaSuccess;
  const ChunkWs ws = chunk_ws_layout(a.b, a.L, a.H);
  BwdMaps tm;
  memset(&tm, 0, sizeof(tm));
  const uint64_t L = (uint64_t)a.L, b = (uint64_t)a.b, H = (uint64_t)a.H, G = (uint64_t)a.G;
  const CUtensorMapDataType bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  // with no tokens the kernel issues no copies (a map needs every extent > 0)
  bool ok = L == 0 || encode_map(&tm.X, bf, a.X, kP, H, L, b, 2, 64, CU_TENSOR_MAP_SWIZZLE_128B) &&
            encode_map(&tm.Y, bf, a.dY, kP, H, L, b, 2, 64, CU_TENSOR_MAP_SWIZZLE_128B) &&
            encode_map(&tm.B, bf, a.B, kN, G, L, b, 2, 64, CU_TENSOR_MAP_SWIZZLE_128B) &&
            encode_map(&tm.C, bf, a.C, kN, G, L, b, 2, 64, CU_TENSOR_MAP_SWIZZLE_128B);
  if (ok && L > 0 && a.theta)
    ok = encode_map(&tm.theta, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, a.theta, kNH, H, L, b, 4, kNH,
                    CU_TENSOR_MAP_SWIZZLE_NONE);
  if (!ok) return cudaErrorInvalidValue;
  const int smem = (int)sizeof(SmT) + 1024;
  cudaError_t e = cudaFuncSetAttribute(bwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  bwd_tc_kernel<<<(unsigned)(a.b * a.H), kT, smem, s>>>(a, ws, tm);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_bwd_chunk_reduce(a, s);
}

cudaError_t read_and_clear_bwd_wait_timeouts(unsigned int* count) {
  unsigned int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(count, g_bwd_tc_wait_timeouts, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_bwd_tc_wait_timeouts, &zero, sizeof(unsigned int));
}

}  // namespace m3ssd
