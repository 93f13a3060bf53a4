// Chunked backward of the Mamba-3 SISO scan in fp32 (N = 128, P = 64, bf16 or
// fp32 inputs), one CTA of 512 threads per (b, h).
//
// The recurrence ("TorchMamba" README, "Math notes", M3 SISO) over a chunk of
// Q = 64 rows -- row 0 the token before the chunk (t0 - 1, the carry-in of the
// trapezoid's beta term), rows 1..63 the chunk's tokens -- reads, with the
// chunk-local decay sums cs_r (cs_0 = 0), cv_u = gamma_u alpha_{u+1} + beta_{u+1}
// (gamma_0 := 0), W(r,u<r) = exp(cs_r - cs_{u+1}) cv_u, W(r,r) = gamma_r and
// W_end(u) = W(63,u):
//   y_r   = exp(cs_r) Cbar_r . h_prev + sum_u W(r,u) (Cbar_r . Bbar_u) x_u + D x_r
//   h_end = exp(cs_63) h_prev + sum_u W_end(u) Bbar_u x_u^T.
// Its adjoint, chunk by chunk in reverse with g = dL/dh_end, E = dY X^T,
// G = Cbar Bbar^T, M = W o G, WE = W o E:
//   dh_prev = exp(cs_63) g + Cbar^T (exp(cs) o dY)
//   dX      = M^T dY + W_end o (Bbar g) + D dY            (row 0 goes to the previous chunk)
//   dCbar   = exp(cs) o (dY h_prev^T) + WE Bbar
//   dBbar   = WE^T Cbar + W_end o (X g^T)                 (row 0 goes to the previous chunk)
//   dW = G o E, dW_end(u) = x_u . (Bbar_u g)   -> decay sums, cv, gamma, beta, logdecay,
// plus exp(cs_r)'s own terms (Cbar_r . h_prev dy_r and <g, h_prev> at r = 63),
// and the rotation adjoints dv = R(phi)^T dvbar, dphi_i, dtheta = suffix sums of dphi.
//
// Pass 1 walks the chunks forward and stores each chunk's starting state (fp32,
// as (p, n)) and angle in the workspace.  Pass 2 walks them in reverse; every
// product is a register-tiled loop over fp32 shared-memory tiles in packed fp32
// pairs, the products with a zero triangle skip it warp by warp, and every
// cross-thread sum runs in a fixed order (warp shuffles, then fixed-order
// shared-memory sums), so the result does not depend on scheduling.  The next
// chunk's inputs are fetched a phase ahead: into registers in pass 1, by
// cp.async into the tiles already free in pass 2 (16-byte aligned inputs; an
// element-wise path otherwise).  The group-shared dB, dC, dbprev0 and dD are
// written per head and summed by a second kernel.
#include "common.cuh"
#include "internal.h"

namespace m3ssd {

namespace {

constexpr int kQ = 64, QT = kQ - 1, kN = 128, kNH = kN / 2, kP = 64, kT = 512;
constexpr int SB = kN + 4;  // row stride of the Bbar / Cbar tiles (floats)
constexpr int SX = kP + 4;  // row stride of the 64-wide tiles
size_t al256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

ChunkWs chunk_ws_layout(int64_t b, int64_t L, int64_t H) {
  const size_t bh = (size_t)(b * H), nC = (size_t)((L + QT - 1) / QT);
  ChunkWs w{};
  size_t o = 0;
  auto take = [&](size_t floats) {
    const size_t r = o;
    o += al256(floats * sizeof(float));
    return r;
  };
  w.hs = take(bh * (nC > 0 ? nC : 1) * kN * kP);
  w.phs = take(bh * (nC > 0 ? nC : 1) * kNH);
  w.dBh = take((size_t)(b * L * H) * kN);
  w.dCh = take((size_t)(b * L * H) * kN);
  w.dbph = take(bh * kN);
  w.dDbh = take(bh);
  w.total = o;
  return w;
}

namespace {

// Shared memory (floats).  The workspace holds each chunk-start state as (p, n).
struct Sm {
  float Bb[kQ * SB];   // B (raw), then Bbar (and W_end o Bbar in pass 1)
  float Cb[kQ * SB];   // C, then Cbar
  float Xs[kQ * SX];   // x rows
  float Ys[kQ * SX];   // dy rows
  float Hp[kP * SB];   // h_prev, transposed: (p, n)
  float Gs[kP * SB];   // g = dL/dh_end, transposed: (p, n)
  float Gm[kQ * SX];   // G, then M, then dphi
  float Em[kQ * SX];   // E, then WE
  float Vt[kQ * SX];   // theta (r, i), then the angles phi (r, i)
  float cs[kQ], al[kQ], ga[kQ], be[kQ], cv[kQ], ecs[kQ], wend[kQ];
  float dcsA[kQ], dcsB[kQ], dcv[kQ], dga[kQ], dwend[kQ], dcsY[kQ];
  float red[kT / 32 * 4];
  float phi0[kNH];     // angle at the chunk start (phi of row 0)
  float cdx[2][kP];    // dX of row 0 of a chunk (carried back), by chunk parity
  float cdb[2][kN];    // dBbar of row 0 of a chunk, by chunk parity
  float run[kNH];      // sum of dphi over all later tokens
  float misc[8];
};
static_assert(sizeof(Sm) <= 232448, "one CTA's shared memory");

// n consecutive elements from p into out (fp32), in 16-byte loads when vec
template <int n>
__device__ __forceinline__ void ldn(const float* p, bool vec, float* out) {
  if (vec) {
#pragma unroll
    for (int k = 0; k < n / 4; ++k) {
      const float4 v = *reinterpret_cast<const float4*>(p + 4 * k);
      out[4 * k] = v.x;
      out[4 * k + 1] = v.y;
      out[4 * k + 2] = v.z;
      out[4 * k + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int k = 0; k < n; ++k) out[k] = p[k];
  }
}
template <int n>
__device__ __forceinline__ void ldn(const __nv_bfloat16* p, bool vec, float* out) {
  if (vec) {
#pragma unroll
    for (int k = 0; k < n / 8; ++k) {
      const uint4 raw = *reinterpret_cast<const uint4*>(p + 8 * k);
      const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[q]));
        out[8 * k + 2 * q] = f.x;
        out[8 * k + 2 * q + 1] = f.y;
      }
    }
  } else {
#pragma unroll
    for (int k = 0; k < n; ++k) out[k] = __bfloat162float(p[k]);
  }
}
// 16 bytes from global to shared memory without a register round trip; the
// destination is zero-filled when !full (nothing is read then)
__device__ __forceinline__ void cp16(float* smem_dst, const void* gmem_src, bool full) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(
                   (uint32_t)__cvta_generic_to_shared(smem_dst)),
               "l"(gmem_src), "r"(full ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// 8 elements held as raw 16-byte vectors (one for bf16, two for fp32) to fp32
__device__ __forceinline__ void unpack8(const uint4* v, float* out, const __nv_bfloat16*) {
  const uint32_t w[4] = {v[0].x, v[0].y, v[0].z, v[0].w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[q]));
    out[2 * q] = f.x;
    out[2 * q + 1] = f.y;
  }
}
__device__ __forceinline__ void unpack8(const uint4* v, float* out, const float*) {
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    out[4 * k] = __uint_as_float(v[k].x);
    out[4 * k + 1] = __uint_as_float(v[k].y);
    out[4 * k + 2] = __uint_as_float(v[k].z);
    out[4 * k + 3] = __uint_as_float(v[k].w);
  }
}
template <int n>
__device__ __forceinline__ void stn(float* dst, const float* v) {
#pragma unroll
  for (int k = 0; k < n / 4; ++k)
    *reinterpret_cast<float4*>(dst + 4 * k) = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
}

// Packed fp32 pairs (two FMAs an instruction on sm_100).
__device__ __forceinline__ float2 lo2(const float4 v) { return make_float2(v.x, v.y); }
__device__ __forceinline__ float2 hi2(const float4 v) { return make_float2(v.z, v.w); }
__device__ __forceinline__ float2 bc2(float v) { return make_float2(v, v); }
// a . b over four terms, accumulated as two partial sums in the lanes of acc
__device__ __forceinline__ float2 acc4(float2 acc, const float4 a, const float4 b) {
  return __ffma2_rn(hi2(a), hi2(b), __ffma2_rn(lo2(a), lo2(b), acc));
}
__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float2 ld2(const float* p) { return *reinterpret_cast<const float2*>(p); }
__device__ __forceinline__ float comp(const float4 v, int m) {
  return m == 0 ? v.x : m == 1 ? v.y : m == 2 ? v.z : v.w;
}
// sum over the 16 lanes of a half-warp (fixed order)
__device__ __forceinline__ float half_sum(float v) {
#pragma unroll
  for (int o = 1; o < 16; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Sum of v over the CTA in a fixed order (warp shuffles, then warp 0 adds the
// 16 warp sums in order); every thread gets the result.
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

static_assert(kNH == kP, "theta rows share the x-row loop");

template <typename T>
__global__ void __launch_bounds__(kT, 1) bwd_chunk_kernel(BwdArgs a, ChunkWs ws) {
  extern __shared__ __align__(16) unsigned char smraw[];
  Sm& sm = *reinterpret_cast<Sm*>(smraw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t H = a.H, G = a.G, L = a.L;
  const int64_t bh = blockIdx.x, b = bh / H, h = bh % H, g = h / (H / G);
  const int nC = (int)((L + QT - 1) / QT);
  const T* X = static_cast<const T*>(a.X);
  const T* Bg = static_cast<const T*>(a.B);
  const T* Cg = static_cast<const T*>(a.C);
  const T* dY = static_cast<const T*>(a.dY);
  const float Dh = a.D ? a.D[h] : 0.f;
  char* wsb = static_cast<char*>(a.workspace);
  float* hs_ws = reinterpret_cast<float*>(wsb + ws.hs) + bh * (int64_t)nC * kN * kP;
  float* ph_ws = reinterpret_cast<float*>(wsb + ws.phs) + bh * (int64_t)nC * kNH;
  float* dBh = reinterpret_cast<float*>(wsb + ws.dBh);
  float* dCh = reinterpret_cast<float*>(wsb + ws.dCh);
  float* dbph = reinterpret_cast<float*>(wsb + ws.dbph);
  float* dDbh = reinterpret_cast<float*>(wsb + ws.dDbh);

  // ---- the inputs of chunk c: rows r <-> tokens t0 - 1 + r -------------------
  // 16-byte loads where every base pointer allows them (rows are whole multiples)
  const bool vec = ((reinterpret_cast<uintptr_t>(X) | reinterpret_cast<uintptr_t>(Bg) |
                     reinterpret_cast<uintptr_t>(Cg) | reinterpret_cast<uintptr_t>(dY) |
                     reinterpret_cast<uintptr_t>(a.theta)) & 15) == 0;
  auto load_chunk = [&](int c, bool bwd) {
    const int64_t t0 = (int64_t)c * QT - 1;
    const int r = tid >> 3, sg = tid & 7;  // row r, columns 8 sg .. (16 sg .. for N)
    const int64_t t = t0 + r;
    const bool in = t >= 0 && t < L, own = r > 0 && t < L;
    const int64_t th = (b * L + (in ? t : 0)) * H + h, tg = (b * L + (in ? t : 0)) * G + g;
    float xv[8], yv[8], tv[8], bv[16], cv[16];
#pragma unroll
    for (int k = 0; k < 8; ++k) xv[k] = yv[k] = tv[k] = 0.f;
#pragma unroll
    for (int k = 0; k < 16; ++k) bv[k] = cv[k] = 0.f;
    if (in) {
      ldn<8>(X + th * kP + 8 * sg, vec, xv);
      ldn<16>(Bg + tg * kN + 16 * sg, vec, bv);
    } else if (t == -1) {
      if (a.xprev0) ldn<8>(a.xprev0 + bh * kP + 8 * sg, false, xv);
      if (a.bprev0) ldn<16>(a.bprev0 + (b * G + g) * kN + 16 * sg, false, bv);
    }
    if (own && a.theta) ldn<8>(a.theta + th * kNH + 8 * sg, vec, tv);
    if (bwd && own) {
      ldn<8>(dY + th * kP + 8 * sg, vec, yv);
      ldn<16>(Cg + tg * kN + 16 * sg, vec, cv);
    }
    float sc[3] = {0.f, 0.f, 0.f};
    if (tid < kQ) {
      const int rr = tid;
      const int64_t tt = t0 + rr;
      if (rr > 0 && tt < L) {
        const int64_t ts = (b * L + tt) * H + h;
        sc[0] = a.logdecay[ts];
        sc[1] = a.gamma[ts];
        sc[2] = a.beta ? a.beta[ts] : 0.f;
      }
    }
    stn<8>(&sm.Xs[r * SX + 8 * sg], xv);
    stn<8>(&sm.Vt[r * SX + 8 * sg], tv);
    stn<16>(&sm.Bb[r * SB + 16 * sg], bv);
    if (bwd) {
      stn<8>(&sm.Ys[r * SX + 8 * sg], yv);
      stn<16>(&sm.Cb[r * SB + 16 * sg], cv);
    }
    if (tid < kQ) {
      sm.cs[tid] = sc[0];  // the raw logdecay until chunk_scalars
      sm.ga[tid] = sc[1];
      sm.be[tid] = sc[2];
    }
  };

  // ---- the same inputs in two steps when every pointer allows 16-byte loads:
  // fetch() issues the loads into registers a phase ahead, commit() converts
  // and stores them (the chunk-start state and angle too, for the reverse pass)
  constexpr int kXV = (int)sizeof(T) / 2;  // 16-byte vectors in 8 elements
  // fp32 inputs need no conversion: the reverse pass copies them asynchronously
  constexpr bool kRaw = sizeof(T) == 4;
  struct Fetch {
    uint4 x[kXV], y[kXV], bq[2 * kXV], cq[2 * kXV];
    float4 th[2];
    float sc[3], ph;
  };
  auto fetch = [&](int c, bool bwd, Fetch& f) {
    const int64_t t0 = (int64_t)c * QT - 1;
    const int r = tid >> 3, sg = tid & 7;
    const int64_t t = t0 + r;
    const bool in = t >= 0 && t < L, own = r > 0 && t < L;
    const int64_t th = (b * L + (in ? t : 0)) * H + h, tg = (b * L + (in ? t : 0)) * G + g;
    const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
    const float4 zf = make_float4(0.f, 0.f, 0.f, 0.f);
    const uint4* xs = reinterpret_cast<const uint4*>(X + th * kP + 8 * sg);
    const uint4* bs = reinterpret_cast<const uint4*>(Bg + tg * kN + 16 * sg);
    if (!(kRaw && bwd)) {
#pragma unroll
      for (int k = 0; k < kXV; ++k) f.x[k] = in ? xs[k] : z4;
#pragma unroll
      for (int k = 0; k < 2 * kXV; ++k) f.bq[k] = in ? bs[k] : z4;
    }
    if (!bwd) {
      const float4* ts = reinterpret_cast<const float4*>(a.theta + th * kNH + 8 * sg);
      f.th[0] = (own && a.theta) ? ts[0] : zf;
      f.th[1] = (own && a.theta) ? ts[1] : zf;
    }
    if (bwd) {
      if (!kRaw) {
        const uint4* ys = reinterpret_cast<const uint4*>(dY + th * kP + 8 * sg);
        const uint4* cs_ = reinterpret_cast<const uint4*>(Cg + tg * kN + 16 * sg);
#pragma unroll
        for (int k = 0; k < kXV; ++k) f.y[k] = own ? ys[k] : z4;
#pragma unroll
        for (int k = 0; k < 2 * kXV; ++k) f.cq[k] = own ? cs_[k] : z4;
      }
      f.ph = tid < kNH ? ph_ws[(int64_t)c * kNH + tid] : 0.f;
    }
    f.sc[0] = f.sc[1] = f.sc[2] = 0.f;
    if (tid < kQ && tid > 0 && t0 + tid < L) {
      const int64_t ts2 = (b * L + t0 + tid) * H + h;
      f.sc[0] = a.logdecay[ts2];
      f.sc[1] = a.gamma[ts2];
      f.sc[2] = a.beta ? a.beta[ts2] : 0.f;
    }
  };
  auto commit = [&](int c, bool bwd, const Fetch& f) {
    const int64_t t0 = (int64_t)c * QT - 1;
    const int r = tid >> 3, sg = tid & 7;
    float xv[8], bv[16];
    const bool carry = t0 + r == -1;  // the cache's carry-in token (fp32)
    if (!(kRaw && bwd) || carry) {
      unpack8(f.x, xv, X);
      unpack8(f.bq, bv, Bg);
      unpack8(f.bq + kXV, bv + 8, Bg);
      if (carry) {
#pragma unroll
        for (int k = 0; k < 8; ++k) xv[k] = a.xprev0 ? a.xprev0[bh * kP + 8 * sg + k] : 0.f;
#pragma unroll
        for (int k = 0; k < 16; ++k)
          bv[k] = a.bprev0 ? a.bprev0[(b * G + g) * kN + 16 * sg + k] : 0.f;
      }
      stn<8>(&sm.Xs[r * SX + 8 * sg], xv);
      stn<16>(&sm.Bb[r * SB + 16 * sg], bv);
    }
    if (!bwd) {
      *reinterpret_cast<float4*>(&sm.Vt[r * SX + 8 * sg]) = f.th[0];
      *reinterpret_cast<float4*>(&sm.Vt[r * SX + 8 * sg + 4]) = f.th[1];
    } else {
      if (!kRaw) {
        float yv[8], cv[16];
        unpack8(f.y, yv, dY);
        unpack8(f.cq, cv, Cg);
        unpack8(f.cq + kXV, cv + 8, Cg);
        stn<8>(&sm.Ys[r * SX + 8 * sg], yv);
        stn<16>(&sm.Cb[r * SB + 16 * sg], cv);
      }
      if (tid < kNH) sm.phi0[tid] = f.ph;
    }
    if (tid < kQ) {
      sm.cs[tid] = f.sc[0];  // the raw logdecay until chunk_scalars
      sm.ga[tid] = f.sc[1];
      sm.be[tid] = f.sc[2];
    }
  };

  // the reverse pass's theta rows and chunk-start state (16-byte asynchronous
  // copies into tiles that are free from the dh_prev phase on)
  auto async_copy = [&](int c) {
    const int64_t t0 = (int64_t)c * QT - 1;
    const float* hw = hs_ws + (int64_t)c * kN * kP;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int e = tid + kT * k, p = e >> 5, n4 = 4 * (e & 31);
      cp16(&sm.Hp[p * SB + n4], hw + p * kN + n4, true);
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int e = tid + kT * k, r = e >> 4, i4 = 4 * (e & 15);
      const int64_t t = t0 + r;
      const bool ok = a.theta && r > 0 && t < L;
      const float* src = ok ? a.theta + ((b * L + t) * H + h) * kNH + i4 : hw;
      cp16(&sm.Vt[r * SX + i4], src, ok);
    }
    if (kRaw) {
#pragma unroll
      for (int k = 0; k < 2; ++k) {  // X, dY: 64 rows of 16 vectors
        const int e = tid + kT * k, r = e >> 4, p4 = 4 * (e & 15);
        const int64_t t = t0 + r;
        const bool in = t >= 0 && t < L, own = r > 0 && t < L;
        const int64_t th = ((b * L + (in ? t : 0)) * H + h) * kP + p4;
        cp16(&sm.Xs[r * SX + p4], X + th, in);
        cp16(&sm.Ys[r * SX + p4], dY + th, own);
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {  // B, C: 64 rows of 32 vectors
        const int e = tid + kT * k, r = e >> 5, n4 = 4 * (e & 31);
        const int64_t t = t0 + r;
        const bool in = t >= 0 && t < L, own = r > 0 && t < L;
        const int64_t tg = ((b * L + (in ? t : 0)) * G + g) * kN + n4;
        cp16(&sm.Bb[r * SB + n4], Bg + tg, in);
        cp16(&sm.Cb[r * SB + n4], Cg + tg, own);
      }
    }
    cp_commit();
  };

  // ---- chunk scalars: cs (inclusive sums of logdecay), alpha, exp(cs), cv, W_end
  auto chunk_scalars = [&]() {
    if (warp == 0) {
      const float l0 = sm.cs[lane], l1 = sm.cs[lane + 32];
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
      sm.al[lane] = expf(l0);
      sm.al[lane + 32] = expf(l1);
      sm.cs[lane] = s0;
      sm.cs[lane + 32] = s1;
    }
    __syncthreads();
    if (tid < kQ) {
      const int r = tid;
      sm.ecs[r] = expf(sm.cs[r]);
      sm.cv[r] = r < kQ - 1 ? sm.ga[r] * sm.al[r + 1] + sm.be[r + 1] : 0.f;
    }
    __syncthreads();
    if (tid < kQ) {
      const int u = tid;
      sm.wend[u] = u < kQ - 1 ? expf(sm.cs[kQ - 1] - sm.cs[u + 1]) * sm.cv[u] : sm.ga[kQ - 1];
    }
    __syncthreads();
  };

  // ---- angles phi(r, i) = phi0[i] + sum_{k <= r} theta(k, i) in Vt, then the
  // rotations of B (and C) in place
  auto angles_rotate = [&](bool rot_c) {
    {
      const int i = tid & 63, grp = tid >> 6;
      float run_ = 0.f;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int r = 8 * grp + k;
        run_ += sm.Vt[r * SX + i];
        sm.Vt[r * SX + i] = run_;
      }
      sm.Gm[grp * SX + i] = run_;  // segment totals (the Gram tile is free here)
      __syncthreads();
      float base = sm.phi0[i];
      for (int q = 0; q < grp; ++q) base += sm.Gm[q * SX + i];
#pragma unroll
      for (int k = 0; k < 8; ++k) sm.Vt[(8 * grp + k) * SX + i] += base;
      __syncthreads();
    }
    for (int e = tid; e < kQ * kNH; e += kT) {
      const int r = e >> 6, i = e & 63;
      float sn, cs_;
      fast_sincos(sm.Vt[r * SX + i], &sn, &cs_);
      float* bp = &sm.Bb[r * SB + 2 * i];
      const float b0 = bp[0], b1 = bp[1];
      bp[0] = cs_ * b0 - sn * b1;
      bp[1] = sn * b0 + cs_ * b1;
      if (rot_c) {
        float* cp = &sm.Cb[r * SB + 2 * i];
        const float c0 = cp[0], c1 = cp[1];
        cp[0] = cs_ * c0 - sn * c1;
        cp[1] = sn * c0 + cs_ * c1;
      }
    }
    __syncthreads();
  };

  // ---- pass 1: the state and the angle at every chunk start -----------------
  // state tile of a thread: n in nq .. nq + 3, p in cq + 16 j
  const int cq = tid & 15, nq = 4 * (tid >> 4);
  {
    float hreg[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j)
        hreg[i][j] = a.h0 ? a.h0[(bh * kN + nq + i) * kP + cq + 16 * j] : 0.f;
    if (tid < kNH) sm.phi0[tid] = wrap_angle(a.angle0 ? a.angle0[bh * kNH + tid] : 0.f);
    Fetch f;
    if (vec && nC > 0) fetch(0, false, f);
    __syncthreads();
    for (int c = 0; c < nC; ++c) {
      float* hw = hs_ws + (int64_t)c * kN * kP;  // (p, n)
#pragma unroll
      for (int j = 0; j < 4; ++j)
        *reinterpret_cast<float4*>(&hw[(cq + 16 * j) * kN + nq]) =
            make_float4(hreg[0][j], hreg[1][j], hreg[2][j], hreg[3][j]);
      if (tid < kNH) ph_ws[(int64_t)c * kNH + tid] = sm.phi0[tid];
      if (vec)
        commit(c, false, f);
      else
        load_chunk(c, false);
      f = Fetch{};  // consumed: nothing stays live across the chunk's compute
      __syncthreads();
      chunk_scalars();
      angles_rotate(false);
      if (vec && c + 1 < nC) fetch(c + 1, false, f);
      const float eE = sm.ecs[kQ - 1];
      float2 acc[2][4];  // rows (nq + 2 ii, nq + 2 ii + 1), column cq + 16 j
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[0][j] = acc[1][j] = make_float2(0.f, 0.f);
      for (int u = 0; u < kQ; ++u) {
        const float2 w = bc2(sm.wend[u]);
        const float4 bv = ld4(&sm.Bb[u * SB + nq]);
        const float2 bw0 = __fmul2_rn(w, lo2(bv)), bw1 = __fmul2_rn(w, hi2(bv));
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 xv = bc2(sm.Xs[u * SX + cq + 16 * j]);
          acc[0][j] = __ffma2_rn(bw0, xv, acc[0][j]);
          acc[1][j] = __ffma2_rn(bw1, xv, acc[1][j]);
        }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        hreg[0][j] = fmaf(eE, hreg[0][j], acc[0][j].x);
        hreg[1][j] = fmaf(eE, hreg[1][j], acc[0][j].y);
        hreg[2][j] = fmaf(eE, hreg[2][j], acc[1][j].x);
        hreg[3][j] = fmaf(eE, hreg[3][j], acc[1][j].y);
      }
      __syncthreads();  // every read of this chunk's tiles is done
      if (tid < kNH) sm.phi0[tid] = wrap_angle(sm.Vt[(kQ - 1) * SX + tid]);
      __syncthreads();
    }
  }

  // ---- pass 2: the chunks in reverse --------------------------------------
  // tiles of 64-row products: rows r0 = 2 rq, r1 = r0 + 1; the rows of a warp
  // are 4 warp .. 4 warp + 3, which bounds the triangular loops warp-uniformly
  const int rq = tid >> 4, r0 = 2 * rq, r1 = r0 + 1;
  const int wlo = 4 * warp, whi = 4 * warp + 3;
  if (tid < kNH) sm.run[tid] = 0.f;
  if (tid < kP) {
    sm.cdx[0][tid] = 0.f;
    sm.cdx[1][tid] = 0.f;
  }
  if (tid < kN) {
    sm.cdb[0][tid] = 0.f;
    sm.cdb[1][tid] = 0.f;
  }
  for (int e = tid; e < kN * kP; e += kT) {
    const int n = e >> 6, p = e & 63;
    sm.Gs[p * SB + n] = a.dhT ? a.dhT[(bh * kN + n) * kP + p] : 0.f;
  }
  float dDacc = 0.f;
  Fetch f;
  if (vec && nC > 0) {
    fetch(nC - 1, true, f);
    async_copy(nC - 1);
  }
  __syncthreads();

  for (int c = nC - 1; c >= 0; --c) {
    const int cur = c & 1, nxt = cur ^ 1;
    const int64_t t0 = (int64_t)c * QT - 1;  // token of row 0
    auto own = [&](int r) { return r > 0 && t0 + r < L; };
    if (vec) {
      cp_wait_all();  // before commit: the carry-in row overwrites a zero-filled copy
      commit(c, true, f);
      f = Fetch{};  // consumed: nothing stays live across the chunk's compute
    } else {
      float4 hpv[4];  // the chunk-start state, (p, n) float4s
      const float* hw = hs_ws + (int64_t)c * kN * kP;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int idx = tid + kT * k;
        hpv[k] = *reinterpret_cast<const float4*>(&hw[(idx >> 5) * kN + 4 * (idx & 31)]);
      }
      if (tid < kNH) sm.phi0[tid] = ph_ws[(int64_t)c * kNH + tid];
      load_chunk(c, true);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int idx = tid + kT * k;
        *reinterpret_cast<float4*>(&sm.Hp[(idx >> 5) * SB + 4 * (idx & 31)]) = hpv[k];
      }
    }
    __syncthreads();
    chunk_scalars();
    angles_rotate(true);

    // -- G = Cbar Bbar^T and E = dY X^T on the lower triangle, then the mask
    //    gradients of dW = G o E, M = W o G and WE = W o E
    {
      float2 gp[2][4], ep[2][4];  // two partial sums each
#pragma unroll
      for (int j = 0; j < 4; ++j) gp[0][j] = gp[1][j] = ep[0][j] = ep[1][j] = make_float2(0.f, 0.f);
      // columns past the warp's last row are masked out (warp-uniform test)
      const int nj = whi / 16 + 1;
#pragma unroll 2
      for (int k = 0; k < kN; k += 4) {
        const float4 c0 = ld4(&sm.Cb[r0 * SB + k]), c1 = ld4(&sm.Cb[r1 * SB + k]);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (j < nj) {
            const float4 bv = ld4(&sm.Bb[(cq + 16 * j) * SB + k]);
            gp[0][j] = acc4(gp[0][j], c0, bv);
            gp[1][j] = acc4(gp[1][j], c1, bv);
          }
      }
#pragma unroll 2
      for (int k = 0; k < kP; k += 4) {
        const float4 y0 = ld4(&sm.Ys[r0 * SX + k]), y1 = ld4(&sm.Ys[r1 * SX + k]);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (j < nj) {
            const float4 xv = ld4(&sm.Xs[(cq + 16 * j) * SX + k]);
            ep[0][j] = acc4(ep[0][j], y0, xv);
            ep[1][j] = acc4(ep[1][j], y1, xv);
          }
      }
      float gt[2][4], et[2][4];
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          gt[i][j] = gp[i][j].x + gp[i][j].y;
          et[i][j] = ep[i][j].x + ep[i][j].y;
        }
      float rowA[2] = {0.f, 0.f}, colB[4] = {0.f, 0.f, 0.f, 0.f}, colV[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int r = r0 + i;
        const float csr = sm.cs[r];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int u = cq + 16 * j;
          const float dW = gt[i][j] * et[i][j];
          float w = 0.f;
          if (u < r) {
            const float ex = expf(csr - sm.cs[u + 1]);
            w = ex * sm.cv[u];
            rowA[i] = fmaf(dW, w, rowA[i]);
            colB[j] = fmaf(dW, w, colB[j]);
            colV[j] = fmaf(dW, ex, colV[j]);
          } else if (u == r) {
            w = sm.ga[r];
            sm.dga[r] = dW;
          }
          gt[i][j] *= w;  // M
          et[i][j] *= w;  // WE
        }
        rowA[i] = half_sum(rowA[i]);
      }
      if (cq == 0) {
        sm.dcsA[r0] = rowA[0];
        sm.dcsA[r1] = rowA[1];
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        colB[j] += __shfl_xor_sync(0xffffffffu, colB[j], 16);
        colV[j] += __shfl_xor_sync(0xffffffffu, colV[j], 16);
      }
      if (lane < 16) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          sm.Gm[warp * SX + cq + 16 * j] = colB[j];
          sm.Em[warp * SX + cq + 16 * j] = colV[j];
        }
      }
      __syncthreads();
      if (tid < 2 * kQ) {
        const int u = tid & 63;
        const float* src = tid < kQ ? sm.Gm : sm.Em;
        float s = 0.f;
        for (int w = 0; w < kT / 32; ++w) s += src[w * SX + u];
        (tid < kQ ? sm.dcsB : sm.dcv)[u] = s;
      }
      __syncthreads();
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          sm.Gm[(r0 + i) * SX + cq + 16 * j] = gt[i][j];
          sm.Em[(r0 + i) * SX + cq + 16 * j] = et[i][j];
        }
      __syncthreads();
    }

    // -- dX = M^T dY + W_end o (Bbar g) + D dY, and dW_end(u) = x_u . (Bbar_u g)
    {
      float vt[2][4], xt[2][4];
      {
        float2 vp[2][4];
#pragma unroll
        for (int j = 0; j < 4; ++j) vp[0][j] = vp[1][j] = make_float2(0.f, 0.f);
        for (int n = 0; n < kN; n += 4) {
          const float4 b0 = ld4(&sm.Bb[r0 * SB + n]), b1 = ld4(&sm.Bb[r1 * SB + n]);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float4 gv = ld4(&sm.Gs[(cq + 16 * j) * SB + n]);
            vp[0][j] = acc4(vp[0][j], b0, gv);
            vp[1][j] = acc4(vp[1][j], b1, gv);
          }
        }
        float2 xp[4];  // (row r0, row r1) pairs
#pragma unroll
        for (int j = 0; j < 4; ++j) xp[j] = make_float2(0.f, 0.f);
        for (int r = wlo; r < kQ; ++r) {  // M(r, u) = 0 for r < u
          const float2 m = ld2(&sm.Gm[r * SX + r0]);
#pragma unroll
          for (int j = 0; j < 4; ++j) xp[j] = __ffma2_rn(m, bc2(sm.Ys[r * SX + cq + 16 * j]), xp[j]);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          vt[0][j] = vp[0][j].x + vp[0][j].y;
          vt[1][j] = vp[1][j].x + vp[1][j].y;
          xt[0][j] = xp[j].x;
          xt[1][j] = xp[j].y;
        }
      }
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int u = r0 + i;
        const float we = sm.wend[u];
        float dwe = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int p = cq + 16 * j;
          const float xv = sm.Xs[u * SX + p], yv = sm.Ys[u * SX + p];
          dwe = fmaf(xv, vt[i][j], dwe);
          dDacc = fmaf(yv, xv, dDacc);
          float dx = xt[i][j] + fmaf(we, vt[i][j], Dh * yv);
          if (u == kQ - 1) dx += sm.cdx[nxt][p];
          if (u == 0)
            sm.cdx[cur][p] = dx;
          else if (own(u))
            a.dX[((b * L + t0 + u) * H + h) * kP + p] = dx;
        }
        dwe = half_sum(dwe);
        if (cq == 0) sm.dwend[u] = dwe;
      }
    }
    __syncthreads();  // M is dead: the Gram tile takes dphi next

    // -- dCbar = exp(cs) o (dY h_prev^T) + WE Bbar, then its rotation adjoint;
    //    columns 4 cq + 64 (k / 4) + k % 4 of rows r0, r1
    {
      float2 ac[2][4];  // column pairs (n, n + 1) of rows r0, r1
#pragma unroll
      for (int q = 0; q < 4; ++q) ac[0][q] = ac[1][q] = make_float2(0.f, 0.f);
      for (int p = 0; p < kP; p += 4) {
        const float4 y0 = ld4(&sm.Ys[r0 * SX + p]), y1 = ld4(&sm.Ys[r1 * SX + p]);
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const float4 h0 = ld4(&sm.Hp[(p + m) * SB + 4 * cq]);
          const float4 h1 = ld4(&sm.Hp[(p + m) * SB + 4 * cq + 64]);
          const float2 hv[4] = {lo2(h0), hi2(h0), lo2(h1), hi2(h1)};
          const float2 ya = bc2(comp(y0, m)), yb = bc2(comp(y1, m));
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            ac[0][q] = __ffma2_rn(ya, hv[q], ac[0][q]);
            ac[1][q] = __ffma2_rn(yb, hv[q], ac[1][q]);
          }
        }
      }
      // exp(cs_r) Cbar_r . (dY h_prev^T)_r: the h_prev term of d cs_r
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int r = r0 + i;
        const float4 c0 = ld4(&sm.Cb[r * SB + 4 * cq]), c1 = ld4(&sm.Cb[r * SB + 4 * cq + 64]);
        const float2 cv[4] = {lo2(c0), hi2(c0), lo2(c1), hi2(c1)};
        float2 s2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int q = 0; q < 4; ++q) s2 = __ffma2_rn(cv[q], ac[i][q], s2);
        const float s = half_sum(s2.x + s2.y);
        const float e = sm.ecs[r];
        if (cq == 0) sm.dcsY[r] = e * s;
#pragma unroll
        for (int q = 0; q < 4; ++q) ac[i][q] = __fmul2_rn(bc2(e), ac[i][q]);
      }
      for (int u = 0; u <= whi; u += 4) {  // WE(r, u) = 0 for u > r
        const float4 w0 = ld4(&sm.Em[r0 * SX + u]), w1 = ld4(&sm.Em[r1 * SX + u]);
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const float4 b0 = ld4(&sm.Bb[(u + m) * SB + 4 * cq]);
          const float4 b1 = ld4(&sm.Bb[(u + m) * SB + 4 * cq + 64]);
          const float2 bv[4] = {lo2(b0), hi2(b0), lo2(b1), hi2(b1)};
          const float2 wa = bc2(comp(w0, m)), wb = bc2(comp(w1, m));
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            ac[0][q] = __ffma2_rn(wa, bv[q], ac[0][q]);
            ac[1][q] = __ffma2_rn(wb, bv[q], ac[1][q]);
          }
        }
      }
      // dC = R(phi)^T dCbar; dphi_i = Cbar x dCbar (the B part is added below)
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int r = r0 + i;
        const bool ok = own(r);
        const int64_t ro = ((b * L + (ok ? t0 + r : 0)) * H + h) * kN;
#pragma unroll
        for (int k = 0; k < 8; k += 2) {
          const int n = 4 * cq + 64 * (k >> 2) + (k & 3), pi = n >> 1;
          float sn, cs_;
          fast_sincos(sm.Vt[r * SX + pi], &sn, &cs_);
          const float d0 = ac[i][k >> 1].x, d1 = ac[i][k >> 1].y;
          const float v0 = sm.Cb[r * SB + n], v1 = sm.Cb[r * SB + n + 1];
          sm.Gm[r * SX + pi] = ok ? fmaf(d1, v0, -d0 * v1) : 0.f;
          if (ok)
            *reinterpret_cast<float2*>(&dCh[ro + n]) =
                make_float2(fmaf(cs_, d0, sn * d1), fmaf(cs_, d1, -sn * d0));
        }
      }
    }

    // -- dBbar = WE^T Cbar + W_end o (X g^T), the carries of row 0 (this
    //    chunk's carry-in token) and into row 63, then the rotation adjoint
    {
      float2 bp[2][4];  // column pairs (n, n + 1) of rows r0, r1
#pragma unroll
      for (int q = 0; q < 4; ++q) bp[0][q] = bp[1][q] = make_float2(0.f, 0.f);
      for (int p = 0; p < kP; p += 4) {
        const float4 x0 = ld4(&sm.Xs[r0 * SX + p]), x1 = ld4(&sm.Xs[r1 * SX + p]);
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const float4 g0 = ld4(&sm.Gs[(p + m) * SB + 4 * cq]);
          const float4 g1 = ld4(&sm.Gs[(p + m) * SB + 4 * cq + 64]);
          const float2 gv[4] = {lo2(g0), hi2(g0), lo2(g1), hi2(g1)};
          const float2 xa = bc2(comp(x0, m)), xb = bc2(comp(x1, m));
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            bp[0][q] = __ffma2_rn(xa, gv[q], bp[0][q]);
            bp[1][q] = __ffma2_rn(xb, gv[q], bp[1][q]);
          }
        }
      }
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const float2 we = bc2(sm.wend[r0 + i]);
#pragma unroll
        for (int q = 0; q < 4; ++q) bp[i][q] = __fmul2_rn(we, bp[i][q]);
      }
      for (int r = wlo; r < kQ; ++r) {  // WE(r, u) = 0 for r < u
        const float2 w = ld2(&sm.Em[r * SX + r0]);
        const float4 c0 = ld4(&sm.Cb[r * SB + 4 * cq]), c1 = ld4(&sm.Cb[r * SB + 4 * cq + 64]);
        const float2 cv[4] = {lo2(c0), hi2(c0), lo2(c1), hi2(c1)};
        const float2 wa = bc2(w.x), wb = bc2(w.y);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          bp[0][q] = __ffma2_rn(wa, cv[q], bp[0][q]);
          bp[1][q] = __ffma2_rn(wb, cv[q], bp[1][q]);
        }
      }
      float bb[2][8];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int r = r0 + i;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int n = 4 * cq + 64 * (k >> 2) + (k & 3);
          bb[i][k] = (k & 1) ? bp[i][k >> 1].y : bp[i][k >> 1].x;
          if (r == kQ - 1) bb[i][k] += sm.cdb[nxt][n];
          if (r == 0) sm.cdb[cur][n] = bb[i][k];
        }
      }
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int r = r0 + i;
        if (!own(r)) continue;
        const int64_t ro = ((b * L + t0 + r) * H + h) * kN;
#pragma unroll
        for (int k = 0; k < 8; k += 2) {
          const int n = 4 * cq + 64 * (k >> 2) + (k & 3), pi = n >> 1;
          float sn, cs_;
          fast_sincos(sm.Vt[r * SX + pi], &sn, &cs_);
          const float d0 = bb[i][k], d1 = bb[i][k + 1];
          const float v0 = sm.Bb[r * SB + n], v1 = sm.Bb[r * SB + n + 1];
          sm.Gm[r * SX + pi] += fmaf(d1, v0, -d0 * v1);
          *reinterpret_cast<float2*>(&dBh[ro + n]) =
              make_float2(fmaf(cs_, d0, sn * d1), fmaf(cs_, d1, -sn * d0));
        }
      }
    }

    // -- dh_prev = exp(cs_63) g + Cbar^T (exp(cs) o dY) and <g, h_prev>
    float dh[4][4];
    {
      const float eE = sm.ecs[kQ - 1];
      float ghp = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int o = (cq + 16 * j) * SB + nq + i;
          const float gv = sm.Gs[o];
          ghp = fmaf(gv, sm.Hp[o], ghp);
          dh[i][j] = eE * gv;
        }
      float2 dp[2][4];  // rows (nq + 2 ii, nq + 2 ii + 1), column cq + 16 j
#pragma unroll
      for (int j = 0; j < 4; ++j) dp[0][j] = dp[1][j] = make_float2(0.f, 0.f);
      for (int r = 1; r < kQ; ++r) {
        const float2 e = bc2(sm.ecs[r]);
        const float4 cv = ld4(&sm.Cb[r * SB + nq]);
        const float2 cw0 = __fmul2_rn(e, lo2(cv)), cw1 = __fmul2_rn(e, hi2(cv));
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 y = bc2(sm.Ys[r * SX + cq + 16 * j]);
          dp[0][j] = __ffma2_rn(cw0, y, dp[0][j]);
          dp[1][j] = __ffma2_rn(cw1, y, dp[1][j]);
        }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        dh[0][j] += dp[0][j].x;
        dh[1][j] += dp[0][j].y;
        dh[2][j] += dp[1][j].x;
        dh[3][j] += dp[1][j].y;
      }
      block_sum(ghp, sm.red, &sm.misc[0]);  // ends with a barrier: g is free
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) sm.Gs[(cq + 16 * j) * SB + nq + i] = dh[i][j];

    if (vec && c > 0) {  // the inputs of chunk c - 1
      fetch(c - 1, true, f);
      async_copy(c - 1);
    }

    // -- the scalar chain: decay sums -> cv -> gamma, beta, logdecay
    if (warp == 0) {
      const float eE = sm.ecs[kQ - 1];
      float endsum = 0.f;
      float dcsv[2];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int u = lane + 32 * k;
        if (u < kQ - 1) endsum = fmaf(sm.dwend[u], sm.wend[u], endsum);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) endsum += __shfl_xor_sync(0xffffffffu, endsum, o);
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int r = lane + 32 * k;
        float d = sm.dcsA[r] + sm.dcsY[r];
        if (r >= 1) d -= sm.dcsB[r - 1] + sm.dwend[r - 1] * sm.wend[r - 1];
        if (r == kQ - 1) d += endsum + eE * sm.misc[0];
        dcsv[k] = d;
        if (r < kQ - 1) sm.dcv[r] = fmaf(sm.dwend[r], expf(sm.cs[kQ - 1] - sm.cs[r + 1]), sm.dcv[r]);
      }
      __syncwarp();
      // suffix sums of dcs over the chunk's rows
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
      const int i = tid & 63, grp = tid >> 6;
      float tmp[8];
      float s = 0.f;
#pragma unroll
      for (int k = 7; k >= 0; --k) {
        s += sm.Gm[(8 * grp + k) * SX + i];
        tmp[k] = s;
      }
      sm.Em[grp * SX + i] = s;
      __syncthreads();
      float base = sm.run[i];
      for (int q = 7; q > grp; --q) base += sm.Em[q * SX + i];
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
  if (a.dh0)
    for (int e = tid; e < kN * kP; e += kT) {
      const int n = e >> 6, p = e & 63;
      a.dh0[(bh * kN + n) * kP + p] = sm.Gs[p * SB + n];
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
  if (tid == 0) dDbh[bh] = dDs;
}

// Sums over the heads of a group (dB, dC, dbprev0) and over the batch (dD),
// each in a fixed order.
// Item r of the sums after dB, dC: dbprev0 (b, G, N) over the heads of each
// group, then dD (H) over the batch, each in a fixed order.
__device__ void reduce_tail(const BwdArgs& a, const ChunkWs& ws, int64_t r) {
  const int64_t H = a.H, G = a.G, hpg = H / G, nbp = a.b * G * kN;
  const char* wsb = static_cast<const char*>(a.workspace);
  const float* dbph = reinterpret_cast<const float*>(wsb + ws.dbph);
  const float* dDbh = reinterpret_cast<const float*>(wsb + ws.dDbh);
  if (r < nbp) {
    const int64_t nn = r % kN, row = r / kN, gg = row % G, bb = row / G;
    float v = 0.f;
    for (int64_t q = 0; q < hpg; ++q) v += dbph[(bb * H + gg * hpg + q) * kN + nn];
    if (a.dbprev0) a.dbprev0[r] = v;
    return;
  }
  r -= nbp;
  float v = 0.f;
  for (int64_t bb = 0; bb < a.b; ++bb) v += dDbh[bb * H + r];
  if (a.dD) a.dD[r] = v;
}

// dB and dC when both outputs are 16-byte aligned: four columns a thread, the
// loads of eight heads in flight at once; every element is still the sum over
// the heads of its group in head order from zero, as in the kernel below, so
// the results are the same bit for bit.  Then dbprev0 and dD.
__global__ void bwd_chunk_reduce_bc4_kernel(BwdArgs a, ChunkWs ws) {
  constexpr int kC4 = kN / 4, kU = 8;
  const int64_t H = a.H, G = a.G;
  const int hpg = (int)(H / G);
  const char* wsb = static_cast<const char*>(a.workspace);
  const float4* dBh = reinterpret_cast<const float4*>(wsb + ws.dBh);
  const float4* dCh = reinterpret_cast<const float4*>(wsb + ws.dCh);
  float4* dB = reinterpret_cast<float4*>(a.dB);
  float4* dC = reinterpret_cast<float4*>(a.dC);
  const int64_t n4 = a.b * a.L * G * kC4, stride = (int64_t)gridDim.x * blockDim.x;
  auto add = [](float4& s, const float4& v) {
    s.x += v.x;
    s.y += v.y;
    s.z += v.z;
    s.w += v.w;
  };
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
    const int64_t c4 = i % kC4, row = i / kC4, gg = row % G, bt = row / G;
    const float4* pb = dBh + (bt * H + gg * hpg) * kC4 + c4;
    const float4* pc = dCh + (bt * H + gg * hpg) * kC4 + c4;
    float4 sb = make_float4(0.f, 0.f, 0.f, 0.f), sc = sb;
    for (int q0 = 0; q0 < hpg; q0 += kU) {
      float4 vb[kU], vc[kU];
#pragma unroll
      for (int k = 0; k < kU; ++k)
        if (q0 + k < hpg) {
          vb[k] = pb[(int64_t)(q0 + k) * kC4];
          vc[k] = pc[(int64_t)(q0 + k) * kC4];
        }
#pragma unroll
      for (int k = 0; k < kU; ++k)
        if (q0 + k < hpg) {
          add(sb, vb[k]);
          add(sc, vc[k]);
        }
    }
    dB[i] = sb;
    dC[i] = sc;
  }
  const int64_t tail = a.b * G * kN + H;  // dbprev0 and dD
  for (int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; r < tail; r += stride)
    reduce_tail(a, ws, r);
}

// The sums over the heads of each group (dB, dC, dbprev0) and over the batch
// (dD) of the per-head shares, in a fixed order.
__global__ void bwd_chunk_reduce_kernel(BwdArgs a, ChunkWs ws) {
  const int64_t H = a.H, G = a.G, hpg = H / G;
  const char* wsb = static_cast<const char*>(a.workspace);
  const float* dBh = reinterpret_cast<const float*>(wsb + ws.dBh);
  const float* dCh = reinterpret_cast<const float*>(wsb + ws.dCh);
  const int64_t nBC = a.b * a.L * G * kN, nbp = a.b * G * kN;
  const int64_t total = nBC + nbp + H;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
    int64_t r = i;
    if (r < nBC) {  // dB, dC: (b, L, G, N)
      const int64_t nn = r % kN, row = r / kN, gg = row % G, bt = row / G;
      float sb = 0.f, sc = 0.f;
      for (int64_t q = 0; q < hpg; ++q) {
        const int64_t src = (bt * H + gg * hpg + q) * kN + nn;
        sb += dBh[src];
        sc += dCh[src];
      }
      a.dB[r] = sb;
      a.dC[r] = sc;
      continue;
    }
    reduce_tail(a, ws, r - nBC);
  }
}

}  // namespace

bool bwd_chunk_supported(int64_t N, int64_t P) { return N == kN && P == kP; }

size_t bwd_chunk_workspace_bytes(int64_t b, int64_t L, int64_t H) {
  return chunk_ws_layout(b, L, H).total;
}

cudaError_t launch_bwd_chunk(const BwdArgs& a, cudaStream_t s) {
  if (a.b * a.H == 0) return cudaSuccess;
  const ChunkWs ws = chunk_ws_layout(a.b, a.L, a.H);
  const int smem = (int)sizeof(Sm);
  cudaError_t e;
  if (a.bf16) {
    e = cudaFuncSetAttribute(bwd_chunk_kernel<__nv_bfloat16>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    bwd_chunk_kernel<__nv_bfloat16><<<(unsigned)(a.b * a.H), kT, smem, s>>>(a, ws);
  } else {
    e = cudaFuncSetAttribute(bwd_chunk_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem);
    if (e != cudaSuccess) return e;
    bwd_chunk_kernel<float><<<(unsigned)(a.b * a.H), kT, smem, s>>>(a, ws);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_bwd_chunk_reduce(a, s);
}

cudaError_t launch_bwd_chunk_reduce(const BwdArgs& a, cudaStream_t s) {
  const ChunkWs ws = chunk_ws_layout(a.b, a.L, a.H);
  auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
  const int64_t nBC = a.b * a.L * a.G * kN;
  const bool bc4 = nBC > 0 && al16(a.dB) && al16(a.dC);
  if (bc4) {
    const int64_t blocks = (nBC / 4 + 255) / 256;
    const unsigned g4 = (unsigned)(blocks < 148 * 8 ? blocks : 148 * 8);
    bwd_chunk_reduce_bc4_kernel<<<g4, 256, 0, s>>>(a, ws);
    return cudaGetLastError();
  }
  const int64_t total = nBC + a.b * a.G * kN + a.H;
  const int64_t blocks = (total + 255) / 256;
  const unsigned rg = (unsigned)(blocks < 148 * 32 ? (blocks > 0 ? blocks : 1) : 148 * 32);
  bwd_chunk_reduce_kernel<<<rg, 256, 0, s>>>(a, ws);
  return cudaGetLastError();
}

}  // namespace m3ssd
