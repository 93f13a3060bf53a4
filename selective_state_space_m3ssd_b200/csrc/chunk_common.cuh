// Pieces shared by the chunked forwards (bf16 and fp32 inputs): the chunk
// geometry, the 128-byte-swizzled tile offsets, the per-chunk scalars the
// control warp prepares, and small conversion helpers.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace m3ssd {
namespace chunk {

constexpr int Q = 64;       // source rows per chunk (1 carry-in + 63 tokens)
constexpr int QT = Q - 1;   // tokens per chunk
constexpr int NS = 128;     // state size N
constexpr int PD = 64;      // head dim P
constexpr int NH = NS / 2;  // rotation pairs
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kAtom = Q * 128;  // bytes of one 64-element atom of a Q-row tile

// Byte offset of element (r, n) in a Q-row tile of 128 elements a row, stored
// as two 64-element atoms of 128-byte rows with the 16-byte XOR swizzle.
__device__ __forceinline__ uint32_t off2(int r, int n) {
  return (uint32_t)((n >> 6) * kAtom + r * 128 + ((((n & 63) >> 3) ^ (r & 7)) << 4) +
                    ((n & 7) << 1));
}
// Byte offset of element (r, c) in a tile of 64 elements (128 B) a row.
__device__ __forceinline__ uint32_t off1(int r, int c) {
  return (uint32_t)(r * 128 + ((((c >> 3) ^ (r & 7))) << 4) + ((c & 7) << 1));
}

// Per-chunk scalars: decay cumsum (scaled by log2 e), exp(cs), the mask
// coefficients gamma_u alpha_{u+1} + beta_{u+1}, the state weights W(63, u),
// gamma, and exp(cs_63).  Double-buffered: chunk c+1's set is computed while
// chunk c is finishing.
struct ChunkParams {
  float cs2[Q];    // cs_r log2(e)
  float ecs[Q];    // exp(cs_r)
  float cvec[Q];   // gamma_r alpha_{r+1} + beta_{r+1}  (gamma_63 for r = 63)
  float wend[Q];   // W(63, r)
  float gam[Q];    // gamma_r
  float et[Q];     // exp(cs_t - cs_{8 floor(t/8)})
  float fs[224];   // exp(cs_{8k} - cs_{s+1}) cvec_s for s < 8k, at fs_index(k, s)
  float dl[Q];     // Delta_r = logdecay_r / A (the raw-angle variant scales theta by it)
  float eE;        // exp(cs_63)
  float pad[3];
};

// The factor table keeps only the entries below the diagonal blocks: block
// row k = 1..7 holds the 8k columns s < 8k, starting at 4 k (k - 1).
__host__ __device__ constexpr int fs_index(int k, int s) { return 4 * k * (k - 1) + s; }

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}
__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float2 unpack_h2(uint32_t u) {
  return __half22float2(*reinterpret_cast<__half2*>(&u));
}
// v as fp16 high and low parts: hi = fp16(v), lo = fp16(v - hi), two values a word
__device__ __forceinline__ void split_h2(float a, float b, uint32_t& hi, uint32_t& lo) {
  hi = pack_h2(a, b);
  const float2 h = unpack_h2(hi);
  lo = pack_h2(a - h.x, b - h.y);
}

// 2^x by the hardware approximation (relative error about 2^-22; flushes
// results below 2^-126 to zero).  The arguments are differences of fp32 decay
// sums, whose own rounding (about |cs| 2^-24) dominates that error.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// One warp: the scalars of one chunk from its per-row logdecay / beta / gamma
// (rows lane and lane + 32; row 0 and rows past the end hold zeros).
__device__ __forceinline__ void chunk_params(ChunkParams& P, const float (&pld)[2],
                                             const float (&pbe)[2], const float (&pga)[2],
                                             int lane, float inv_a) {
  P.dl[lane] = pld[0] * inv_a;
  P.dl[lane + 32] = pld[1] * inv_a;
  // decay sums in log2 units
  float s0 = pld[0] * kLog2e, s1 = pld[1] * kLog2e;
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
  // the sum at the first row of each 8-row block, and at this lane's own block
  float mk[8];
#pragma unroll
  for (int k = 0; k < 8; ++k)
    mk[k] = __shfl_sync(0xffffffffu, k < 4 ? s0 : s1, (8 * k) & 31);
  const float mown0 = __shfl_sync(0xffffffffu, s0, lane & ~7);
  const float mown1 = __shfl_sync(0xffffffffu, s1, lane & ~7);
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int r = lane + 32 * k;
    const float ld_next = k == 0 ? (lane < 31 ? ld_dn0 : ld_32) : ld_dn1;
    const float be_next = k == 0 ? (lane < 31 ? be_dn0 : be_32) : be_dn1;
    const float cs_next = k == 0 ? (lane < 31 ? cs_dn0 : cs_32) : cs_dn1;
    P.cs2[r] = cs[k];
    P.ecs[r] = ex2(cs[k]);
    P.gam[r] = pga[k];
    P.et[r] = ex2(cs[k] - (k == 0 ? mown0 : mown1));
    float cv;
    if (r < Q - 1) {
      cv = pga[k] * ex2(ld_next * kLog2e) + be_next;
      P.wend[r] = ex2(cs_end - cs_next) * cv;
    } else {
      cv = pga[k];
      P.wend[r] = cv;
    }
    P.cvec[r] = cv;
    // the factor table, for the blocks k2 strictly below this column's block
#pragma unroll
    for (int k2 = 0; k2 < 8; ++k2)
      if (8 * k2 > r) P.fs[fs_index(k2, r)] = ex2(mk[k2] - cs_next) * cv;
  }
  if (lane == 0) P.eE = ex2(cs_end);
}

}  // namespace chunk
}  // namespace m3ssd
