// Sequence split of the chunked bf16 forward (N = 128, P = 64) for launches
// with too few (b, h) sequences to fill the GPU (one CTA walks a sequence's
// chunks in order, so b H sequences keep at most b H SMs busy).
//
// The recurrence ("TorchMamba" README, "Math notes", M3 SISO) is linear in the
// state, so a sequence cut into segments k = 0 .. S-1 (k covering the tokens
// [s_k, e_k)) has
//     h_{e_k - 1} = exp(D_k) h_{s_k - 1} + R(Phi_{e_k - 1}) hloc_k,
// where D_k is the segment's summed log decay, Phi_{e_k - 1} the absolute angle
// at its last token, and hloc_k the state the segment builds from a zero start,
// written in the frame of its last token: every row u of the segment enters
// rotated by minus the angle summed over the tokens after u, and weighted by
// its trapezoid coefficient and the decay from u + 1 to the segment end.  So
// every weight is at most 1 and every angle is referred to the segment end,
// which lets the pass walk the segment's chunks from the last to the first and
// keep both running sums (the decay after the chunk, the angle after it) as
// scalars.  The row-0 carry-in of each chunk brings the beta term of the
// chunk's first token, as in the chunked forward.
//
// Three launches on the caller's stream:
//   1. fwd_seg_state_kernel: one CTA per (b, h, k < S - 1), hloc_k as one
//      tensor-core accumulation Bbar^T (w o X) over the segment's chunks
//      (M = 128 n, N = 64 p, K = 64 rows a chunk; fp16 operands, fp32 in TMEM),
//      plus D_k (log2 units) and the segment's angle sum;
//   2. fwd_seg_combine_kernel: one CTA per (b, h), the start state and angle
//      of segments 1 .. S-1 from the relation above (in fp32);
//   3. the chunked forward with one CTA per (b, h, k) from those starts.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cstring>

#include "chunk_common.cuh"
#include "common.cuh"
#include "internal.h"
#include "tc5.cuh"

namespace m3ssd {

__device__ unsigned int g_seg_wait_timeouts;

namespace {

using namespace chunk;

constexpr int kCtrlWarp = 8;                    // the control warp
constexpr int kThreads = 32 * (kCtrlWarp + 1);  // 8 compute warps + 1 control warp
constexpr uint32_t kTmemCols = 64;              // hloc: 128 lanes (n) x 64 columns (p)
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr uint32_t kIdescS = tc5::idesc_f16(128, 64, true, true);
constexpr int kMinSegChunks = 8;  // a segment holds at least this many chunks

// Raw inputs of one chunk (double-buffered: the next-but-one chunk's copies land
// while this one is processed).
struct SegIn {
  float theta[Q][NH];     // fp32, no swizzle
  uint8_t B[2 * kAtom];   // bf16, two 64-element atoms, 128-byte swizzle
  uint8_t X[Q * 128];     // bf16, 128-byte swizzle
};
struct SegSmem {
  SegIn in[2];
  uint8_t Bb[2 * kAtom];  // Bbar in fp16: the product's A operand (MN-major)
  uint8_t wx[Q * 128];    // w o X in fp16: its B operand (MN-major)
  float w[2][Q];          // each row's weight toward the segment end
  float segtot[8][NH];
  float tha[2][NH];       // angle summed over the chunks after this one, reduced
  uint64_t lmbar[2];      // copies of input buffer 0 / 1
  uint64_t smbar;         // one phase per issued product
  uint32_t tmem;
  uint32_t err;
};
static_assert(2 * (sizeof(SegSmem) + 1024 + 1024) <= 233472, "two CTAs per SM");
static_assert(offsetof(SegSmem, Bb) % 1024 == 0 && offsetof(SegSmem, wx) % 1024 == 0,
              "operand tiles on 1024-byte boundaries");
static_assert(sizeof(SegIn) % 1024 == 0 && offsetof(SegIn, B) % 1024 == 0 &&
                  offsetof(SegIn, X) % 1024 == 0,
              "copy destinations on 1024-byte boundaries");

struct SegMaps {
  CUtensorMap theta;  // fp32 (pair, head, token, batch), box 64 x 1 x 64 x 1
  CUtensorMap B;      // bf16 (n, group, token, batch), box 64 x 1 x 64 x 1, 128-byte swizzle
  CUtensorMap X;      // bf16 (p, head, token, batch), same box and swizzle
};

// Workspace regions (floats), for U = b H (S - 1) segment-pass units.
struct SegWs {
  size_t hl, hs, psi, as, dt, total;  // offsets in floats; total in bytes
};
SegWs seg_ws(int64_t b, int64_t H, int nseg) {
  const size_t U = (size_t)(b * H) * (size_t)(nseg - 1);
  SegWs w;
  w.hl = 0;
  w.hs = w.hl + U * NS * PD;
  w.psi = w.hs + U * NS * PD;
  w.as = w.psi + U * NH;
  w.dt = w.as + U * NH;
  w.total = (w.dt + ((U + 63) / 64) * 64) * sizeof(float);
  return w;
}

template <bool ROT>
__global__ void __launch_bounds__(kThreads, 2)
    fwd_seg_state_kernel(FwdArgs a, const __grid_constant__ SegMaps tm, float* hl, float* psi,
                         float* dt) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw_addr = tc5::saddr(smem_raw);
  SegSmem& sm = *reinterpret_cast<SegSmem*>(smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool ctrl = warp == kCtrlWarp;
  const bool ctrl_lead = tid == kCtrlWarp * 32;
  const int64_t H = a.H, L = a.L, G = a.G;
  const int nsa = a.nseg - 1;  // segment-pass units of a sequence
  const int64_t bh = blockIdx.x / nsa;
  const int k = (int)(blockIdx.x - bh * nsa);
  const int64_t b = bh / H, h = bh % H, g = h / (H / G);
  const int c_lo = k * a.segc, n = a.segc;  // full chunks; processing step i takes chunk c_lo + n - 1 - i
  const bool has_theta = ROT && a.theta != nullptr;
  const uint32_t bytes = (has_theta ? 16384u : 0u) + 16384u + 8192u;

  auto issue = [&](int i) {  // control thread: the copies of step i into buffer i & 1
    const int c = c_lo + n - 1 - i;
    SegIn& in = sm.in[i & 1];
    uint64_t* mb = &sm.lmbar[i & 1];
    const int t = c * QT - 1;
    tc5::mbar_arrive_expect_tx(mb, bytes);
    if (has_theta) tc5::tma_load_4d(tc5::saddr(&in.theta[0][0]), &tm.theta, mb, 0, (int)h, t, (int)b);
    tc5::tma_load_4d(tc5::saddr(in.B), &tm.B, mb, 0, (int)g, t, (int)b);
    tc5::tma_load_4d(tc5::saddr(in.B) + kAtom, &tm.B, mb, 64, (int)g, t, (int)b);
    tc5::tma_load_4d(tc5::saddr(in.X), &tm.X, mb, 0, (int)h, t, (int)b);
  };
  // the control warp keeps logdecay / beta / gamma of rows lane and lane + 32 of
  // the next step's chunk in registers
  float pld[2], pbe[2], pga[2];
  auto load_params = [&](int i) {
    const int c = c_lo + n - 1 - i;
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
      const int r = lane + 32 * kk;
      const int64_t t = (int64_t)c * QT - 1 + r;
      const bool ok = r > 0 && t < L;  // row 0 (carry-in) has a = gamma = beta = 0 here
      const int64_t idx = (b * L + (ok ? t : 0)) * H + h;
      pld[kk] = ok ? a.logdecay[idx] : 0.f;
      pga[kk] = ok ? a.gamma[idx] : 0.f;
      pbe[kk] = (ok && a.beta) ? a.beta[idx] : 0.f;
    }
  };
  // control warp: the weights of step i's rows toward the segment end,
  //   w_u = 2^(dacc + cs_63 - cs_{u+1}) (gamma_u alpha_{u+1} + beta_{u+1}),  u < 63,
  //   w_63 = 2^dacc gamma_63,
  // with cs the chunk's decay cumsum and dacc the decay of the chunks after it
  // (log2 units; row 0 has gamma = 0, so w_0 is the beta term of row 1); then
  // dacc += cs_63
  float dacc = 0.f;
  auto params = [&](int i) {
    float s0 = pld[0] * kLog2e, s1 = pld[1] * kLog2e;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float u0 = __shfl_up_sync(0xffffffffu, s0, o);
      const float u1 = __shfl_up_sync(0xffffffffu, s1, o);
      if (lane >= o) { s0 += u0; s1 += u1; }
    }
    s1 += __shfl_sync(0xffffffffu, s0, 31);
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
    float* w = sm.w[i & 1];
    // row lane (its successor is row lane + 1, lane 31's is row 32)
    const float ld_n = lane < 31 ? ld_dn0 : ld_32, be_n = lane < 31 ? be_dn0 : be_32;
    const float cs_n = lane < 31 ? cs_dn0 : cs_32;
    w[lane] = ex2(dacc + cs_end - cs_n) * (pga[0] * ex2(ld_n * kLog2e) + be_n);
    // row lane + 32 (row 63 keeps its own gamma term only)
    w[lane + 32] = lane < 31 ? ex2(dacc + cs_end - cs_dn1) * (pga[1] * ex2(ld_dn1 * kLog2e) + be_dn1)
                             : ex2(dacc) * pga[1];
    dacc += cs_end;
  };

  if (warp == 0) tc5::tmem_alloc(&sm.tmem, kTmemCols);
  if (ctrl_lead) {
    tc5::mbar_init(&sm.lmbar[0], 1);
    tc5::mbar_init(&sm.lmbar[1], 1);
    tc5::mbar_init(&sm.smbar, 1);
    tc5::fence_mbar_init();
    sm.err = 0;
  }
  if (tid < NH) sm.tha[0][tid] = 0.f;
  __syncthreads();
  if (ctrl_lead) {
    issue(0);
    if (n > 1) issue(1);
  }
  if (ctrl) {
    load_params(0);
    params(0);
    if (n > 1) load_params(1);
  }
  // the sequence's first chunk: row 0 is the cache's previous token
  const bool first_chunk_here = k == 0;
  const float bp0 = (first_chunk_here && tid < NS && a.bprev0) ? a.bprev0[(b * G + g) * NS + tid] : 0.f;
  const float xp0 = (first_chunk_here && tid < PD && a.xprev0) ? a.xprev0[bh * PD + tid] : 0.f;
  const bool patch_row0 = first_chunk_here && (a.bprev0 != nullptr || a.xprev0 != nullptr);
  tc5::fence_before_sync();
  __syncthreads();
  tc5::fence_after_sync();
  const uint32_t tmem = sm.tmem;
  const uint32_t aBb = tc5::saddr(sm.Bb), aWX = tc5::saddr(sm.wx);

  for (int i = 0; i < n; ++i) {
    const uint32_t lpar = (uint32_t)((i >> 1) & 1);
    SegIn& in = sm.in[i & 1];
    if (tid == 0 && !tc5::mbar_wait(&sm.lmbar[i & 1], lpar, kWaitLimitNs)) sm.err = 1;
    tc5::fence_before_sync();
    __syncthreads();  // S1: step i's inputs landed; step i-1's scalars ready
    tc5::fence_after_sync();
    if (sm.err) {
      // let the copies and the product in flight land before TMEM is freed
      (void)tc5::mbar_wait(&sm.lmbar[i & 1], lpar, kWaitLimitNs);
      if (i + 1 < n)  // step i+1's copies were issued with step i-1's product (or first)
        (void)tc5::mbar_wait(&sm.lmbar[(i + 1) & 1], (uint32_t)(((i + 1) >> 1) & 1), kWaitLimitNs);
      if (i > 0) (void)tc5::mbar_wait(&sm.smbar, (uint32_t)((i - 1) & 1), kWaitLimitNs);
      break;
    }

    if (ctrl) {
      // ===================== control warp ======================================
      if (i + 1 < n) {
        params(i + 1);
        if (i + 2 < n) load_params(i + 2);
      }
      __syncthreads();  // S3: Bbar and w o X of step i ready
      if (ctrl_lead) {
        tc5::fence_after_sync();
        const uint64_t dA = tc5::desc_sw128(aBb, kAtom, 1024), dW = tc5::desc_sw128(aWX, kAtom, 1024);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint64_t kofs = (uint64_t)(j * (2048 >> 4));
          tc5::mma_bf16(tmem, dA + kofs, dW + kofs, kIdescS, i > 0 || j > 0);
        }
        tc5::commit(&sm.smbar);
        // every raw input of buffer i & 1 has been read: refill it
        if (i + 2 < n) issue(i + 2);
      }
      continue;
    }

    // ===================== compute warps (0..7) =================================
    if (patch_row0 && i == n - 1) {  // the sequence's chunk 0
      if (tid < NS) *reinterpret_cast<__nv_bfloat16*>(in.B + off2(0, tid)) = __float2bfloat16_rn(bp0);
      if (tid < PD) *reinterpret_cast<__nv_bfloat16*>(in.X + off1(0, tid)) = __float2bfloat16_rn(xp0);
    }
    // -- angles toward the segment end: thread (lane, warp) owns the pairs 2 lane,
    // 2 lane + 1 in rows 8 warp .. 8 warp + 7 (row 0's own theta is not summed)
    float2 psi_l[8], run = make_float2(0.f, 0.f);
    if (has_theta) {
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        if (warp > 0 || kk > 0)
          run = __fadd2_rn(run, *reinterpret_cast<const float2*>(&in.theta[8 * warp + kk][2 * lane]));
        psi_l[kk] = run;
      }
      *reinterpret_cast<float2*>(&sm.segtot[warp][2 * lane]) = run;
    }
    // (the patch of row 0 and every read of theta come before the barrier)
    asm volatile("bar.sync 1, %0;" ::"n"(32 * kCtrlWarp) : "memory");
    float2 suf = make_float2(0.f, 0.f);  // theta summed after this warp's rows
    if (has_theta) {
      suf = *reinterpret_cast<const float2*>(&sm.tha[i & 1][2 * lane]);
#pragma unroll
      for (int s2 = 1; s2 < 8; ++s2)
        if (s2 > warp) suf = __fadd2_rn(suf, *reinterpret_cast<const float2*>(&sm.segtot[s2][2 * lane]));
      if (tid < NH) {
        float tot = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) tot += sm.segtot[w][tid];
        sm.tha[(i + 1) & 1][tid] = wrap_angle(sm.tha[i & 1][tid] + tot);
      }
    }
    // the previous step's product has read Bbar and w o X
    if (i > 0 && !tc5::mbar_wait(&sm.smbar, (uint32_t)((i - 1) & 1), kWaitLimitNs)) sm.err = 1;
    tc5::fence_after_sync();
    // -- Bbar = R(-angle after the row) B in fp16
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const int r = 8 * warp + kk;
      const uint32_t o = off2(r, 4 * lane);
      const uint2 bw2 = *reinterpret_cast<const uint2*>(in.B + o);
      float2 bre = make_float2(__uint_as_float(bw2.x << 16), __uint_as_float(bw2.y << 16));
      float2 bim = make_float2(__uint_as_float(bw2.x & 0xffff0000u), __uint_as_float(bw2.y & 0xffff0000u));
      if (has_theta) {
        // minus (theta after row r inside the chunk + theta of the later chunks)
        const float2 after = __fadd2_rn(suf, make_float2(run.x - psi_l[kk].x, run.y - psi_l[kk].y));
        float s0, c0, s1, c1;
        __sincosf(-after.x, &s0, &c0);
        __sincosf(-after.y, &s1, &c1);
        const float2 cr = make_float2(c0, c1), sr = make_float2(s0, s1);
        const float2 nsr = make_float2(-s0, -s1);
        const float2 re2 = __ffma2_rn(nsr, bim, __fmul2_rn(cr, bre));
        const float2 im2 = __ffma2_rn(cr, bim, __fmul2_rn(sr, bre));
        bre = re2;
        bim = im2;
      }
      *reinterpret_cast<uint2*>(sm.Bb + o) = make_uint2(pack_h2(bre.x, bim.x), pack_h2(bre.y, bim.y));
    }
    {  // w o X in fp16: row tid / 4, 16 elements a thread
      const int r = tid >> 2;
      const float we = sm.w[i & 1][r];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int ch = 2 * (tid & 3) + q;
        const uint32_t o = (uint32_t)(r * 128 + ((ch ^ (r & 7)) << 4));
        const uint4 xw = *reinterpret_cast<const uint4*>(in.X + o);
        const uint32_t w4[4] = {xw.x, xw.y, xw.z, xw.w};
        uint32_t outw[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
          outw[j] = pack_h2(we * __uint_as_float(w4[j] << 16), we * __uint_as_float(w4[j] & 0xffff0000u));
        *reinterpret_cast<uint4*>(sm.wx + o) = make_uint4(outw[0], outw[1], outw[2], outw[3]);
      }
    }
    tc5::fence_proxy_async();
    tc5::fence_before_sync();
    __syncthreads();  // S3
  }

  // ---- hloc, the angle sum and the decay sum of the segment ---------------------
  if (!sm.err && !ctrl && n > 0) {
    if (!tc5::mbar_wait(&sm.smbar, (uint32_t)((n - 1) & 1), kWaitLimitNs)) sm.err = 1;
    tc5::fence_after_sync();
    const int n_row = 32 * (warp & 3) + lane, cb = 32 * ((warp >> 2) & 1);
    uint32_t sv[32];
    tc5::ld_32x32b_x32(tmem + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)cb, sv);
    tc5::wait_ld();
    float4* dst = reinterpret_cast<float4*>(hl + ((size_t)blockIdx.x * NS + n_row) * PD + cb);
#pragma unroll
    for (int j = 0; j < 8; ++j)
      dst[j] = make_float4(__uint_as_float(sv[4 * j]), __uint_as_float(sv[4 * j + 1]),
                           __uint_as_float(sv[4 * j + 2]), __uint_as_float(sv[4 * j + 3]));
    if (tid < NH) psi[(size_t)blockIdx.x * NH + tid] = has_theta ? sm.tha[n & 1][tid] : 0.f;
  }
  if (ctrl && lane == 0) dt[blockIdx.x] = dacc;
  tc5::fence_before_sync();
  __syncthreads();
  if (tid == 0 && sm.err) atomicAdd(&g_seg_wait_timeouts, 1u);
  if (warp == 0) tc5::tmem_dealloc(tmem, kTmemCols);
}

// Start state and angle of segments 1 .. S-1 of sequence blockIdx.y:
//   h_start(k) = 2^dt(k-1) h_start(k-1) + R(Phi_end(k-1)) hloc(k-1),
//   Phi_end(k-1) = Phi_start(k-1) + psi(k-1) = Phi_start(k),
// from h_start(0) = h0 (or 0) and Phi_start(0) = angle0 (or 0).  A thread takes
// the rows (2 i, 2 i + 1) of one column p: item blockIdx.x 256 + threadIdx.x.
__global__ void __launch_bounds__(256)
    fwd_seg_combine_kernel(FwdArgs a, const float* hl, const float* psi, const float* dt,
                           float* hs, float* as, bool rot) {
  const int64_t bh = blockIdx.y;
  const int nsa = a.nseg - 1;
  {
    const int e = blockIdx.x * blockDim.x + threadIdx.x;  // < NH PD by the grid
    const int i = e / PD, p = e % PD;
    float re = a.h0 ? a.h0[(bh * NS + 2 * i) * PD + p] : 0.f;
    float im = a.h0 ? a.h0[(bh * NS + 2 * i + 1) * PD + p] : 0.f;
    float phi = (rot && a.angle0) ? wrap_angle(a.angle0[bh * NH + i]) : 0.f;
    for (int k = 1; k <= nsa; ++k) {
      const size_t u = (size_t)bh * nsa + (k - 1);
      const float dec = exp2f(dt[u]);
      const float lre = hl[(u * NS + 2 * i) * PD + p], lim = hl[(u * NS + 2 * i + 1) * PD + p];
      float nre, nim;
      if (rot) {
        phi = wrap_angle(phi + psi[u * NH + i]);
        float s, c;
        sincosf(phi, &s, &c);
        nre = fmaf(dec, re, c * lre - s * lim);
        nim = fmaf(dec, im, s * lre + c * lim);
      } else {
        nre = fmaf(dec, re, lre);
        nim = fmaf(dec, im, lim);
      }
      re = nre;
      im = nim;
      hs[(u * NS + 2 * i) * PD + p] = re;
      hs[(u * NS + 2 * i + 1) * PD + p] = im;
      if (p == 0) as[u * NH + i] = phi;
    }
  }
}

}  // namespace

int current_device_sms() {
  // remembered per device (the forward asks on every call)
  static std::atomic<int> known[64];
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return 0;
  }
  if (dev >= 0 && dev < 64 && (n = known[dev].load(std::memory_order_relaxed)) > 0) return n;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    (void)cudaGetLastError();
    return 0;
  }
  if (dev >= 0 && dev < 64) known[dev].store(n, std::memory_order_relaxed);
  return n;
}

SplitPlan fwd_split_plan(int64_t b, int64_t L, int64_t H, int sms) {
  SplitPlan p{1, 0};
  const int64_t units = b * H;
  const int64_t nC = (L + QT - 1) / QT;
  if (units <= 0 || sms <= 0 || nC < 2 * kMinSegChunks) return p;
  // two chunk-walking CTAs fit on an SM; a split pays when it at least triples
  // the CTAs that run at once
  int64_t S = (2 * (int64_t)sms) / units;
  if (S < 3) return p;
  S = S < nC / kMinSegChunks ? S : nC / kMinSegChunks;
  if (S < 2) return p;
  const int64_t segc = (nC + S - 1) / S;
  const int64_t nseg = (nC + segc - 1) / segc;
  if (nseg < 2) return p;
  p.nseg = (int)nseg;
  p.segc = (int)segc;
  return p;
}

size_t fwd_split_workspace_bytes(int64_t b, int64_t H, const SplitPlan& p) {
  if (p.nseg < 2) return 0;
  return seg_ws(b, H, p.nseg).total;
}

cudaError_t launch_fwd_split(const FwdArgs& a0, const SplitPlan& p, void* workspace,
                             cudaStream_t s) {
  FwdArgs a = a0;
  a.nseg = p.nseg;
  a.segc = p.segc;
  const SegWs w = seg_ws(a.b, a.H, p.nseg);
  float* ws = static_cast<float*>(workspace);
  float *hl = ws + w.hl, *hs = ws + w.hs, *psi = ws + w.psi, *as = ws + w.as, *dt = ws + w.dt;
  const bool rot = a.theta != nullptr || a.angle0 != nullptr;

  SegMaps tm;
  memset(&tm, 0, sizeof(tm));
  const uint64_t L = (uint64_t)a.L, b = (uint64_t)a.b, H = (uint64_t)a.H, G = (uint64_t)a.G;
  bool ok = encode_map(&tm.B, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.B, NS, G, L, b, 2, 64,
                       CU_TENSOR_MAP_SWIZZLE_128B) &&
            encode_map(&tm.X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.X, PD, H, L, b, 2, 64,
                       CU_TENSOR_MAP_SWIZZLE_128B);
  if (ok && a.theta)
    ok = encode_map(&tm.theta, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, a.theta, NH, H, L, b, 4, NH,
                    CU_TENSOR_MAP_SWIZZLE_NONE);
  if (!ok) return cudaErrorInvalidValue;
  const size_t smem = sizeof(SegSmem) + 1024;
  const unsigned units = (unsigned)(a.b * a.H * (p.nseg - 1));
  cudaError_t e;
  if (rot) {
    e = cudaFuncSetAttribute(fwd_seg_state_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    fwd_seg_state_kernel<true><<<units, kThreads, smem, s>>>(a, tm, hl, psi, dt);
  } else {
    e = cudaFuncSetAttribute(fwd_seg_state_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    fwd_seg_state_kernel<false><<<units, kThreads, smem, s>>>(a, tm, hl, psi, dt);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  fwd_seg_combine_kernel<<<dim3(NH * PD / 256, (unsigned)(a.b * a.H)), 256, 0, s>>>(a, hl, psi, dt,
                                                                                   hs, as, rot);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  a.hseg = hs;
  a.aseg = as;
  return launch_fwd_chunk(a, s);
}

cudaError_t read_and_clear_seg_wait_timeouts(unsigned int* count) {
  const unsigned int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(count, g_seg_wait_timeouts, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_seg_wait_timeouts, &zero, sizeof(unsigned int));
}

}  // namespace m3ssd
