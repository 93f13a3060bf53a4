// The per-row chunk scalars of the chunked MIMO forwards (bf16 and fp32 inputs):
// a chunk of 64 rows holds 64 / R tokens, row R j + rho for token j and rank rho,
// and every row takes its token's decay sums, trapezoid weights and mask factors.
#pragma once

#include <stdint.h>

#include "chunk_common.cuh"

namespace m3ssd {
namespace mchunk {

using chunk::Q;
using chunk::ex2;
using chunk::fs_index;
using chunk::kLog2e;

// Per-row chunk scalars (each row takes its token's values), double-buffered.
struct MParams {
  float cs2[Q];    // decay sum of the row's token, log2 units
  float csn2[Q];   // the same for the next token
  float ecs[Q];    // exp(cs)
  float cvec[Q];   // gamma_j alpha_{j+1} + beta_{j+1}  (gamma of the last token)
  float wend[Q];   // W(last token, j)
  float gam[Q];    // gamma_j (0 for the carry-in token)
  float et[Q];     // exp(cs_row - cs at the first row of the row's 8-row block)
  float fs[224];   // exp(cs_{8k} - cs_next(s)) cvec_s for rows s < 8k, at fs_index(k, s)
  float eE;        // exp(cs of the last token)
  float pad[3];
};


// One warp (lane = chunk-local token j): the per-row scalars of one chunk from the
// per-token logdecay / beta / gamma (token 0 and tokens past the end hold zeros).
template <int R>
__device__ __forceinline__ void chunk_params(MParams& P, float ld, float be, float ga, int lane) {
  constexpr int TQ = Q / R;
  float s = ld * kLog2e;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float u = __shfl_up_sync(0xffffffffu, s, o);
    if (lane >= o) s += u;
  }
  const float cs_end = __shfl_sync(0xffffffffu, s, TQ - 1);
  const float ld_n = __shfl_down_sync(0xffffffffu, ld, 1);
  const float be_n = __shfl_down_sync(0xffffffffu, be, 1);
  const float cs_n = __shfl_down_sync(0xffffffffu, s, 1);
  const bool last = lane >= TQ - 1;
  const float cv = last ? ga : ga * ex2(ld_n * kLog2e) + be_n;
  const float we = last ? ga : ex2(cs_end - cs_n) * cv;
  const float csn = last ? s : cs_n;
  float mk[8];  // decay sum at the first row of each 8-row block
#pragma unroll
  for (int k = 0; k < 8; ++k) mk[k] = __shfl_sync(0xffffffffu, s, (8 * k) / R);
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int r = lane + 32 * k, j = r / R;
    const float cs_r = __shfl_sync(0xffffffffu, s, j);
    const float csn_r = __shfl_sync(0xffffffffu, csn, j);
    const float cv_r = __shfl_sync(0xffffffffu, cv, j);
    const float we_r = __shfl_sync(0xffffffffu, we, j);
    const float ga_r = __shfl_sync(0xffffffffu, ga, j);
    const float mb = __shfl_sync(0xffffffffu, s, (r & ~7) / R);
    P.cs2[r] = cs_r;
    P.csn2[r] = csn_r;
    P.ecs[r] = ex2(cs_r);
    P.cvec[r] = cv_r;
    P.wend[r] = we_r;
    P.gam[r] = ga_r;
    P.et[r] = ex2(cs_r - mb);
#pragma unroll
    for (int k2 = 0; k2 < 8; ++k2)
      if (8 * k2 > r) P.fs[fs_index(k2, r)] = ex2(mk[k2] - csn_r) * cv_r;
  }
  if (lane == 0) P.eE = ex2(cs_end);
}

}  // namespace mchunk
}  // namespace m3ssd
